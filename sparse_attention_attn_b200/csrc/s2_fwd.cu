// S2-Attn forward for sm_100a: tcgen05 UMMA with TMEM accumulators, TMA-fed
// Q and K/V rings, online softmax in fp32 with one query row per thread.
//
// A persistent CTA (one per SM) walks a static list of items; an item is the
// pair of adjacent query tiles (2i, 2i+1) of one rolled group of one
// (batch, head).  The key/value tiles of an item run from the start of the
// group up to the diagonal of its second tile; tiles above the diagonal and
// outside the group are never touched (LongQLoRA community post, section 03:
// attention only inside each group; section 04: causal next-token objective).
// Every K/V tile feeds both query tiles, so one load serves 256 query rows.
//
// Warp roles (320 threads):
//   warp 0      TMA producer: Q tiles into a 3-slot ring (the next item's
//               tiles are fetched while the current item runs), K_j / V_j
//               into a KV ring.
//   warp 1      TMEM owner and UMMA issuer: S_A = Q_A K_j^T, S_B = Q_B K_j^T,
//               O_A += P_A V_j, O_B += P_B V_j, in the order S_A(0) S_B(0)
//               PV_A(0) S_A(1) PV_B(0) S_B(1) PV_A(1) ... so the tensor core
//               works on one tile while the softmax of the other runs.
//   warps 2..5  softmax warpgroup A (query tile 2i), warps 6..9 warpgroup B
//               (tile 2i+1): one thread per query row; S from TMEM, running
//               max and sum, P (bf16) written back over S in two 64-key
//               halves (P V on the first starts while the second is being
//               computed), O rescaled in TMEM only when the running max grows
//               by more than 2^8; epilogue: O / l staged in the tile's Q slot
//               and written by TMA stores, lse by the threads.
//
// The issuer starts the next item's S for a warpgroup as soon as that
// warpgroup's last P V of the current item is issued.  TMEM (512 columns):
// S_A [0,128), S_B [128,256) (P over their first 64 columns),
// O_A [256, 256+D), O_B [256+D, 256+2D).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "s2_common.cuh"
#include "s2_ptx.cuh"

namespace s2 {

// KVS: slots of the K/V ring (K and V tiles share it: K0 V0 K1 V1 ...), the
// pipeline depth the per-shape plan selects (4 at head dim 128, 4-8 at 64).
// At least 4: the issuer starts the next item's first S (which needs the
// next item's K_0) before it releases the current item's last V / K tiles, so
// K_0's slot must be one released earlier -- with 4 slots it is K_ta's, the
// last K tile both warpgroups have finished with.
template <int D, int KVS>
struct FwdCfg {
  static constexpr int BM = kTile, BN = kTile;
  static constexpr int QSLOTS = 3;                  // Q ring: two tiles per item, one ahead
  static constexpr int KVSLOTS = KVS;
  static constexpr int ATOM_BYTES = kTile * 128;    // one 64-column slab of a 128-row tile
  static constexpr int TILE_BYTES = kTile * D * 2;  // one 128-row tile of Q, K or V
  static constexpr int OFF_KV = QSLOTS * TILE_BYTES;
  static constexpr int SMEM_BYTES = OFF_KV + KVSLOTS * TILE_BYTES + 1024;  // + alignment slack
  static constexpr uint32_t TM_O = 256;
  static constexpr int THREADS = 320;
  static_assert(SMEM_BYTES <= 232448 - 512, "shared memory");
  static_assert(KVSLOTS >= 4, "the next item's K_0 needs a slot released before the item ends");
};

template <int D, int KVS>
__global__ void __launch_bounds__(320, 1)
    s2_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                  const FwdArgs a) {
  using C = FwdCfg<D, KVS>;
  constexpr int NQ = C::QSLOTS, NS = C::KVSLOTS;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) uint64_t bar_qfull[NQ], bar_qempty[NQ], bar_full[NS], bar_empty[NS],
      bar_s[2], bar_plo[2], bar_p[2], bar_o[2], bar_ofree[2], bar_drain;
  __shared__ uint32_t tmem_slot;
  __shared__ uint32_t abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Dims& d = a.d;
  WaitCtx wc{&abort_flag, a.status, a.wait_limit_ns};

  const uint32_t sQ = smem_u32(smem);
  auto q_addr = [&](int s) { return sQ + s * C::TILE_BYTES; };
  auto kv_addr = [&](int s) { return sQ + C::OFF_KV + s * C::TILE_BYTES; };

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < NQ; ++s) {
      mbar_init(smem_u32(&bar_qfull[s]), 1);
      mbar_init(smem_u32(&bar_qempty[s]), 4);  // the four warps whose O went out through the slot
    }
    for (int s = 0; s < NS; ++s) {
      mbar_init(smem_u32(&bar_full[s]), 1);
      mbar_init(smem_u32(&bar_empty[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bar_s[i]), 1);
      mbar_init(smem_u32(&bar_plo[i]), 4);    // P keys 0..63 written: one arrival per warp of the warpgroup
      mbar_init(smem_u32(&bar_p[i]), 4);      // P keys 64..127 written
      mbar_init(smem_u32(&bar_o[i]), 1);
      mbar_init(smem_u32(&bar_ofree[i]), 4);
    }
    mbar_init(smem_u32(&bar_drain), 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // (whole warp converged; one elected lane issues the copies)
    if (elect_one()) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
    __syncwarp();
    int qu = 0;  // Q-ring uses so far (two per item)
    int L = 0;   // KV-ring loads so far
    // Q use qu: query tile t of item it, or (absent second tile) a plain
    // arrival that completes the slot's phase without data.
    auto load_q = [&](const FwdItem& it, int t, bool present) -> bool {
      const int s = qu % NQ, r = qu / NQ;
      if (r > 0 && !warp_wait(smem_u32(&bar_qempty[s]), (r - 1) & 1, wc, 10)) return false;
      const int row = original_row(d, it.g * d.G + t * kTile, it.sh);
      if (present && !in_bounds(a.status, row, d.N - kTile + 1, 41)) present = false;
      if (elect_one()) {
        if (present) {
          mbar_arrive_expect_tx(smem_u32(&bar_qfull[s]), C::TILE_BYTES);
          for (int c = 0; c < D / 64; ++c)
            tma_load_4d(q_addr(s) + c * C::ATOM_BYTES, &tmQ, smem_u32(&bar_qfull[s]), c * 64, it.h,
                        row, it.b);
        } else {
          mbar_arrive(smem_u32(&bar_qfull[s]));
        }
      }
      __syncwarp();
      ++qu;
      return true;
    };
    auto load_kv = [&](const FwdItem& it, int j, bool is_v) -> bool {
      const int s = L % NS, r = L / NS;
      if (r > 0 && !warp_wait(smem_u32(&bar_empty[s]), (r - 1) & 1, wc, 11)) return false;
      // key tile j: a listed historical tile first (HGA mode), then the group's own
      int row = j < it.nh ? it.hist[j] * kTile : original_row_kv(d, it.g * d.G + (j - it.nh) * kTile, it.sh);
      if (!in_bounds(a.status, row, d.Nk - kTile + 1, 42)) row = 0;  // debug build: load a valid tile instead
      if (elect_one()) {
        mbar_arrive_expect_tx(smem_u32(&bar_full[s]), C::TILE_BYTES);
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(kv_addr(s) + c * C::ATOM_BYTES, is_v ? &tmV : &tmK, smem_u32(&bar_full[s]),
                      c * 64, it.kvh, row, it.b);
      }
      __syncwarp();
      ++L;
      return true;
    };
    FwdCursor cur;
    cur.first(a.sched);
    bool ok = true;
    if (cur.valid) {
      FwdItem it = fwd_item(d, cur.unit, cur.i, a.hist);
      ok = load_q(it, it.ta, true) && load_q(it, it.ta + 1, it.has_b);
      bool qb_pending = false;  // this item's second Q tile is still to come
      while (ok && cur.valid) {
        FwdCursor nx = cur;
        nx.next(a.sched);
        const FwdItem itn = fwd_item(d, nx.valid ? nx.unit : cur.unit, nx.valid ? nx.i : cur.i, a.hist);
        // The next item's first Q tile goes into the slot the previous item's
        // second tile freed: fetched once this item is under way.  An item's
        // second Q tile goes into the slot whose tile's O the epilogue stages
        // at the end of the previous item: fetched after this item's first
        // K/V tiles, so those never wait for that epilogue.
        const int jq = min(2, it.nkv - 1);
        for (int j = 0; ok && j < it.nkv; ++j) {
          ok = load_kv(it, j, false) && load_kv(it, j, true);
          if (ok && j == 0 && qb_pending) {
            ok = load_q(it, it.ta + 1, it.has_b);
            qb_pending = false;
          }
          if (ok && j == jq && nx.valid) ok = load_q(itn, itn.ta, true);
        }
        qb_pending = nx.valid;
        cur = nx;
        it = itn;
      }
    }
    if (*wc.abort && lane == 0) {
      // never leave copies in flight into shared memory: wait (bounded) for
      // the last fill of every slot
      for (int s = 0; s < NQ && s < qu; ++s) drain_wait(smem_u32(&bar_qfull[s]), ((qu - 1 - s) / NQ) & 1);
      for (int s = 0; s < NS && s < L; ++s) drain_wait(smem_u32(&bar_full[s]), ((L - 1 - s) / NS) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer
    // (whole warp converged; one elected lane issues each batch)
    const uint32_t idS = make_idesc_bf16(128, C::BN, 0, 0);  // Q K-major, K K-major
    const uint32_t idO = make_idesc_bf16(128, D, 0, 1);      // P from TMEM, V MN-major
    const uint64_t dQ0 = make_sdesc_sw128(q_addr(0), 16, 1024);              // K-major
    const uint64_t dK0 = make_sdesc_sw128(kv_addr(0), 16, 1024);             // K-major
    const uint64_t dV0 = make_sdesc_sw128(kv_addr(0), C::ATOM_BYTES, 1024);  // MN-major
    auto commit = [&](uint64_t* bar) {
      if (elect_one()) umma_commit(smem_u32(bar));
      __syncwarp();
    };
    auto wait_full = [&](int Lx) { return warp_wait(smem_u32(&bar_full[Lx % NS]), (Lx / NS) & 1, wc, 20); };
    // A Q slot is normally released by the epilogue that staged its tile's O
    // there (four warps); an item without a second tile releases that slot here.
    auto release_q = [&](int slot) {
      for (int i = 0; i < 4; ++i) commit(&bar_qempty[slot]);
    };
    // S_wg = Q(slot qs) K(load Lk)^T
    auto issue_s = [&](int wg, int qs, int Lk) {
      tc_fence_after();
      const uint64_t dq = sdesc_advance(dQ0, qs * C::TILE_BYTES);
      const uint64_t dk = sdesc_advance(dK0, (Lk % NS) * C::TILE_BYTES);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::ATOM_BYTES + (kk & 3) * 32;
          umma_ss(tmem + wg * 128, sdesc_advance(dq, off), sdesc_advance(dk, off), idS, kk > 0);
        }
        umma_commit(smem_u32(&bar_s[wg]));
      }
      __syncwarp();
    };
    int L = 0, n = 0, np[2] = {0, 0};  // ring loads and items consumed, P halves received per warpgroup
    // O_wg (+)= P_wg V(load Lv), keys 64h .. 64h+63 (the half of P that
    // has arrived); the second half completes the product (bar_o)
    auto issue_pv = [&](int wg, int Lv, int h, bool acc) {
      tc_fence_after();
      const uint64_t dv = sdesc_advance(dV0, (Lv % NS) * C::TILE_BYTES);
      if (elect_one()) {
#pragma unroll
        for (int kq = 0; kq < C::BN / 32; ++kq) {
          const int kk = h * (C::BN / 32) + kq;
          umma_ts(tmem + C::TM_O + wg * D, tmem + wg * 128 + kk * 8, sdesc_advance(dv, kk * 2048), idO,
                  acc || kk > 0);
        }
        if (h == 1) umma_commit(smem_u32(&bar_o[wg]));
      }
      __syncwarp();
    };
    // P_wg(j) V_j: the first half as soon as P keys 0..63 are in TMEM
    // (V_j's arrival is waited for once: by warpgroup A's P V, or by B's
    // when A does not use tile j)
    auto pv = [&](int wg, int Lv, int j, bool first_of_item, bool need_v) -> bool {
      if (!warp_wait(smem_u32(&bar_plo[wg]), np[wg] & 1, wc, wg == 0 ? 22 : 24) ||
          (first_of_item && n > 0 && !warp_wait(smem_u32(&bar_ofree[wg]), (n - 1) & 1, wc, wg == 0 ? 23 : 25)) ||
          (need_v && !wait_full(Lv)))
        return false;
      issue_pv(wg, Lv, 0, j > 0);
      if (!warp_wait(smem_u32(&bar_p[wg]), np[wg] & 1, wc, wg == 0 ? 28 : 29)) return false;
      issue_pv(wg, Lv, 1, true);
      ++np[wg];
      return true;
    };
    bool pre = false;  // this item's first S_A / S_B were issued at the end of the previous item
    FwdCursor cur;
    cur.first(a.sched);
    bool ok = true;
    while (ok && cur.valid) {
      const FwdItem it = fwd_item(d, cur.unit, cur.i, a.hist);
      FwdCursor nx = cur;
      nx.next(a.sched);
      const FwdItem itn = fwd_item(d, nx.valid ? nx.unit : cur.unit, nx.valid ? nx.i : cur.i, a.hist);
      const int uA = 2 * n, uB = uA + 1, sA = uA % NQ, sB = uB % NQ;
      const int sAn = (uA + 2) % NQ, sBn = (uB + 2) % NQ;  // the next item's Q slots
      const int lastA = it.lastA, lastB = it.lastB;
      const int L0 = L;  // K_j is load L0 + 2j, V_j load L0 + 2j + 1
      const int L0n = L0 + 2 * it.nkv;
      if (!pre) {
        ok = warp_wait(smem_u32(&bar_qfull[sA]), (uA / NQ) & 1, wc, 21) && wait_full(L0) &&
             warp_wait(smem_u32(&bar_qfull[sB]), (uB / NQ) & 1, wc, 21);
        if (!ok) break;
        issue_s(0, sA, L0);
        if (it.has_b) issue_s(1, sB, L0);
        else release_q(sB);
        commit(&bar_empty[L0 % NS]);
      } else if (!it.has_b) {
        // the absent second tile's Q slot (filled without data) goes back here,
        // once every UMMA of the previous item is issued: waiting for it any
        // earlier could hold up that item's second-tile work, whose released
        // K/V slots the producer needs before it reaches this slot
        if (!(ok = warp_wait(smem_u32(&bar_qfull[sB]), (uB / NQ) & 1, wc, 26))) break;
        release_q(sB);
      }
      // The next item's first scores are computed as soon as this item's
      // last P V of the same warpgroup has been issued (it reads P out of the
      // S buffer before the new S overwrites it), so a warpgroup moves on to
      // the next item without waiting for the other one to finish this item.
      auto start_next_a = [&]() -> bool {
        if (!nx.valid) return true;
        if (!warp_wait(smem_u32(&bar_qfull[sAn]), ((uA + 2) / NQ) & 1, wc, 26) || !wait_full(L0n)) return false;
        issue_s(0, sAn, L0n);
        if (!itn.has_b) commit(&bar_empty[L0n % NS]);  // its K_0 has no second reader
        return true;
      };
      auto start_next_b = [&]() -> bool {
        if (!nx.valid || !itn.has_b) return true;
        if (!warp_wait(smem_u32(&bar_qfull[sBn]), ((uB + 2) / NQ) & 1, wc, 27)) return false;
        issue_s(1, sBn, L0n);
        commit(&bar_empty[L0n % NS]);
        return true;
      };
      for (int j = 0; ok && j < it.nkv; ++j) {
        const int Lv = L0 + 2 * j + 1, Lk1 = L0 + 2 * j + 2;
        if (j <= lastA) {
          if (!(ok = pv(0, Lv, j, j == 0, true))) break;
          if (j > lastB) commit(&bar_empty[Lv % NS]);
          if (j + 1 <= lastA) {
            if (!wait_full(Lk1)) { ok = false; break; }
            issue_s(0, sA, Lk1);
            if (j + 1 > lastB) commit(&bar_empty[Lk1 % NS]);
          } else if (!(ok = start_next_a() && (lastB >= 0 || start_next_b()))) {
            break;
          }
        }
        if (j <= lastB) {
          if (!(ok = pv(1, Lv, j, j == 0, j > lastA))) break;
          commit(&bar_empty[Lv % NS]);
          if (j + 1 <= lastB) {
            if (j + 1 > lastA && !wait_full(Lk1)) { ok = false; break; }
            issue_s(1, sB, Lk1);
            commit(&bar_empty[Lk1 % NS]);
          } else if (!(ok = start_next_b())) {
            break;
          }
        }
      }
      L = L0n;
      ++n;
      pre = nx.valid;
      cur = nx;
    }
    // every issued UMMA completes before TMEM is released
    if (elect_one()) {
      umma_commit(smem_u32(&bar_drain));
      drain_wait(smem_u32(&bar_drain), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    // warpgroup wg owns query tile ta + wg of every item; thread = query row
    const int wg = (warp - 2) >> 2;
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + wg * 128;
    const uint32_t tO = tmem + lane_off + C::TM_O + wg * D;
    const float sl2 = a.scale_log2;
    int ns = 0, no = 0;  // S and PV phases of this warpgroup so far
    int n_item = 0;      // items walked (the Q-ring use of this warpgroup's tile is 2 n_item + wg)
    FwdCursor cur;
    cur.first(a.sched);
    bool ok = true;
    while (ok && cur.valid) {
      const FwdItem it = fwd_item(d, cur.unit, cur.i, a.hist);
      const int t = it.ta + wg;
      const int jlast = wg == 0 ? it.lastA : it.lastB;  // the diagonal key tile when causal
      if (wg == 0 || it.has_b) {
        float m_run = 0.f, l_run = 0.f;
        for (int j = 0; j <= jlast; ++j) {
          ok = warp_wait(smem_u32(&bar_s[wg]), ns & 1, wc, 30);
          if (!ok) break;
          ++ns;
          tc_fence_after();
          uint32_t sr[4][32];
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, sr[c]);
          tmem_wait_ld();
          if (d.causal && j == jlast) {  // diagonal tile: keys after the query are masked
#pragma unroll
            for (int c = 0; c < 128; ++c)
              if (c > row) sr[c >> 5][c & 31] = __float_as_uint(neg_inf());
          }
          // row max with three-input max instructions (exact: the same
          // value as pairwise maxima), four independent chains
          float m4[4] = {neg_inf(), neg_inf(), neg_inf(), neg_inf()};
#pragma unroll
          for (int c = 0; c < 128; c += 8) {
#pragma unroll
            for (int u = 0; u < 4; ++u)
              m4[u] = fmax3(m4[u], __uint_as_float(sr[c >> 5][(c & 31) + 2 * u]),
                            __uint_as_float(sr[c >> 5][(c & 31) + 2 * u + 1]));
          }
          const float mx = fmax3(fmaxf(m4[0], m4[1]), m4[2], m4[3]) * sl2;
          float alpha = 1.f;
          bool resc = false;
          if (j == 0) {
            m_run = mx;
          } else if (mx > m_run + 8.f) {
            alpha = ex2_approx(m_run - mx);
            m_run = mx;
            resc = true;
          }
          // P (bf16) over the first 64 columns of S, in two halves so the
          // issuer can start P V on keys 0..63 while keys 64..127 are being
          // computed; every S column of this thread's row was read above.
          // Each half goes out in two 16-column pieces, which keeps the
          // softmax within the register budget (no spills)
          uint32_t pk[16];
          float rs = softmax_row32(sr[0], sl2, m_run, pk);
          tmem_st16(tS, pk);
          rs += softmax_row32(sr[1], sl2, m_run, pk);
          tmem_st16(tS + 16, pk);
          if (__any_sync(0xffffffffu, resc)) {
            // rescale O (it holds P_{j-1} V_{j-1} once that UMMA has completed)
            // before P_j V_j accumulates onto it
            ok = warp_wait(smem_u32(&bar_o[wg]), (no - 1) & 1, wc, 31);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t o[32];
              tmem_ld32(tO + c * 32, o);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
              tmem_st32(tO + c * 32, o);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&bar_plo[wg]));
          rs += softmax_row32(sr[2], sl2, m_run, pk);
          tmem_st16(tS + 32, pk);
          rs += softmax_row32(sr[3], sl2, m_run, pk);
          tmem_st16(tS + 48, pk);
          l_run = l_run * alpha + rs;
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&bar_p[wg]));
          ++no;
        }
        // ---------------------------------------------------------- epilogue
        if (ok) {
          ok = warp_wait(smem_u32(&bar_o[wg]), (no - 1) & 1, wc, 32);
        }
        if (!ok) break;
        tc_fence_after();
        uint32_t o[D / 32][32];
#pragma unroll
        for (int c = 0; c < D / 32; ++c) tmem_ld32(tO + c * 32, o[c]);
        tmem_wait_ld();
        // O is in registers: the issuer may start the next item's P V
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bar_ofree[wg]));
        const float inv_l = 1.f / l_run;
        const int tq0 = original_row(d, it.g * d.G + t * kTile, it.sh);  // the tile never wraps
        const int tq = tq0 + row;
        // O (bf16) of this warp's 32 rows into the tile's Q slot, whose last
        // reader (this tile's last S) has completed: 128-byte swizzled rows in
        // the TMA layout, then one TMA store per 64-column slab; the slot goes
        // back to the producer once the stores have read it
        const int qs = (2 * n_item + wg) % NQ;
        const uint32_t stage = q_addr(qs) + row * 128;
        const uint32_t sw = static_cast<uint32_t>(row & 7);
#pragma unroll
        for (int sl = 0; sl < D / 64; ++sl) {
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const uint32_t* src = &o[2 * sl + (ch >> 2)][(ch & 3) * 8];
            st_shared_v4(stage + sl * C::ATOM_BYTES + ((ch ^ sw) << 4),
                         pack_bf16x2(__uint_as_float(src[0]) * inv_l, __uint_as_float(src[1]) * inv_l),
                         pack_bf16x2(__uint_as_float(src[2]) * inv_l, __uint_as_float(src[3]) * inv_l),
                         pack_bf16x2(__uint_as_float(src[4]) * inv_l, __uint_as_float(src[5]) * inv_l),
                         pack_bf16x2(__uint_as_float(src[6]) * inv_l, __uint_as_float(src[7]) * inv_l));
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          for (int sl = 0; sl < D / 64; ++sl)
            tma_store_4d(&tmO, q_addr(qs) + sl * C::ATOM_BYTES + quarter * 32 * 128, sl * 64, it.h, tq0 + quarter * 32,
                         it.b);
          bulk_commit_group();
          bulk_wait_read_all();
          mbar_arrive(smem_u32(&bar_qempty[qs]));
        }
        __syncwarp();
        const long long li = (static_cast<long long>(it.b) * d.H + it.h) * d.N + tq;
        if (in_bounds(a.status, li, static_cast<long long>(d.B) * d.H * d.N, 40))
          a.lse[li] = (m_run + __log2f(l_run)) * 0.69314718055994530942f;
      } else {
        // no second tile in this item: keep the O-free phases in step
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bar_ofree[wg]));
      }
      ++n_item;
      cur.next(a.sched);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D, int KVS>
cudaError_t launch_fwd_slots(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const CUtensorMap& to, const FwdArgs& a, int num_sms, cudaStream_t stream) {
  using C = FwdCfg<D, KVS>;
  cudaError_t ea = cudaFuncSetAttribute(s2_fwd_kernel<D, KVS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        C::SMEM_BYTES);
  if (ea != cudaSuccess) return ea;
  const int grid = a.sched.n < num_sms ? a.sched.n : num_sms;
  prof_before(stream, kKernelFwd);
  s2_fwd_kernel<D, KVS><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, to, a);
  cudaError_t e = cudaGetLastError();
  prof_after(stream);
  return e;
}

// kv_slots: depth of the K/V ring, 4 at head dim 128 and 4, 6 or 8 at head
// dim 64 (at least 4, see FwdCfg; at most what fits in shared memory beside
// the three Q slots); anything else is an invalid value.
template <int D>
cudaError_t launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& to, const FwdArgs& a, int num_sms, cudaStream_t stream, int kv_slots) {
  if constexpr (D == 128) {
    switch (kv_slots) {
      case 4: return launch_fwd_slots<D, 4>(tq, tk, tv, to, a, num_sms, stream);
      default: return cudaErrorInvalidValue;
    }
  } else {
    switch (kv_slots) {
      case 4: return launch_fwd_slots<D, 4>(tq, tk, tv, to, a, num_sms, stream);
      case 6: return launch_fwd_slots<D, 6>(tq, tk, tv, to, a, num_sms, stream);
      case 8: return launch_fwd_slots<D, 8>(tq, tk, tv, to, a, num_sms, stream);
      default: return cudaErrorInvalidValue;
    }
  }
}

template cudaError_t launch_fwd<64>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                    const CUtensorMap&, const FwdArgs&, int, cudaStream_t, int);
template cudaError_t launch_fwd<128>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                     const CUtensorMap&, const FwdArgs&, int, cudaStream_t, int);

}  // namespace s2
