// S2-Attn forward with 64-key tiles and double-buffered scores (sm_100a).
//
// The same items, schedule and warp roles as s2_fwd.cu (a persistent CTA walks
// pairs of adjacent 128-row query tiles of one rolled group; warp 0 loads,
// warp 1 issues the UMMAs, warpgroups A and B each own one query tile, one
// query row per thread), but the keys advance 64 at a time and each
// warpgroup's 128 TMEM score columns hold two 64-column buffers.  S(j+1) is
// computed into the other buffer while the softmax works on S(j), so a
// warpgroup's softmax never waits for the P V of its previous tile and the
// next S behind it: with 128-key tiles P is written over the only score
// buffer, and the next S can only start once P V has read it, which chains
// softmax -> P V -> S -> softmax.  The price is an SS UMMA with N = 64 for
// Q K^T (shared-memory bound, about 51 instead of 32 cycles per K = 16 step)
// and twice as many softmax steps per key; the online softmax (running max,
// lazy O rescale by more than 2^8) treats every 64-key tile as a step.
//
// TMEM: S_A [0,128) = buffers [0,64) and [64,128), S_B [128,256), P (bf16)
// over the first 32 columns of its buffer; O_A [256, 256+D), O_B [256+D, 256+2D).
// Issue order per 64-key tile j: P V_A(j), S_A(j+2), P V_B(j), S_B(j+2); the
// next item's first two S of a warpgroup take the places of S(n) and S(n+1).
// The K/V ring needs at least 8 slots of 64 rows: when warpgroup A starts the
// next item, up to six of this item's K/V tiles are still in use.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "s2_common.cuh"
#include "s2_ptx.cuh"

namespace s2 {

template <int D, int KVS>
struct Fwd64Cfg {
  static constexpr int BN = 64;
  static constexpr int QSLOTS = 3;
  static constexpr int KVSLOTS = KVS;
  static constexpr int Q_ATOM = kTile * 128;    // one 64-column slab of a 128-row Q tile
  static constexpr int KV_ATOM = BN * 128;      // one 64-column slab of a 64-row K / V tile
  static constexpr int Q_BYTES = kTile * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int OFF_KV = QSLOTS * Q_BYTES;
  static constexpr int SMEM_BYTES = OFF_KV + KVSLOTS * KV_BYTES + 1024;
  static constexpr uint32_t TM_O = 256;
  static constexpr int THREADS = 320;
  static_assert(SMEM_BYTES <= 232448 - 512, "shared memory");
  static_assert(KVSLOTS >= 8, "the next item's first K tiles need slots beside this item's last six");
};

template <int D, int KVS>
__global__ void __launch_bounds__(320, 1)
    s2_fwd64_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                    const FwdArgs a) {
  using C = Fwd64Cfg<D, KVS>;
  constexpr int NQ = C::QSLOTS, NS = C::KVSLOTS;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) uint64_t bar_qfull[NQ], bar_qempty[NQ], bar_full[NS], bar_empty[NS], bar_s[2][2],
      bar_p[2][2], bar_o[2], bar_ofree[2], bar_drain;
  __shared__ uint32_t tmem_slot;
  __shared__ uint32_t abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Dims& d = a.d;
  WaitCtx wc{&abort_flag, a.status, a.wait_limit_ns};
  const uint32_t sQ = smem_u32(smem);
  auto q_addr = [&](int s) { return sQ + s * C::Q_BYTES; };
  auto kv_addr = [&](int s) { return sQ + C::OFF_KV + s * C::KV_BYTES; };
  // 64-key tiles of an item for warpgroup wg (two per 128-key tile up to its diagonal)
  auto n_tiles = [&](const FwdItem& it, int wg) {
    return wg == 0 ? 2 * (it.lastA + 1) : (it.has_b ? 2 * (it.lastB + 1) : 0);
  };

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
      mbar_init(smem_u32(&bar_s[i][0]), 1);
      mbar_init(smem_u32(&bar_s[i][1]), 1);
      // P written into buffer 0 / 1: one arrival per warp of the warpgroup.  One
      // barrier per buffer: the softmax may run a tile ahead of the issuer (both
      // scores of the next two tiles can be ready), so a single barrier could
      // complete two phases before the issuer looks at the first
      mbar_init(smem_u32(&bar_p[i][0]), 4);
      mbar_init(smem_u32(&bar_p[i][1]), 4);
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
    if (elect_one()) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
    __syncwarp();
    int qu = 0;  // Q-ring uses so far (two per item)
    int L = 0;   // KV-ring loads so far
    auto load_q = [&](const FwdItem& it, int t, bool present) -> bool {
      const int s = qu % NQ, r = qu / NQ;
      if (r > 0 && !warp_wait(smem_u32(&bar_qempty[s]), (r - 1) & 1, wc, 10)) return false;
      const int row = original_row(d, it.g * d.G + t * kTile, it.sh);
      if (present && !in_bounds(a.status, row, d.N - kTile + 1, 41)) present = false;
      if (elect_one()) {
        if (present) {
          mbar_arrive_expect_tx(smem_u32(&bar_qfull[s]), C::Q_BYTES);
          for (int c = 0; c < D / 64; ++c)
            tma_load_4d(q_addr(s) + c * C::Q_ATOM, &tmQ, smem_u32(&bar_qfull[s]), c * 64, it.h, row, it.b);
        } else {
          mbar_arrive(smem_u32(&bar_qfull[s]));
        }
      }
      __syncwarp();
      ++qu;
      return true;
    };
    // 64-row key / value tile j of an item: half (j & 1) of 128-key tile j >> 1
    // (a listed historical tile first in HGA mode, then the group's own)
    auto load_kv = [&](const FwdItem& it, int j, bool is_v) -> bool {
      const int s = L % NS, r = L / NS;
      if (r > 0 && !warp_wait(smem_u32(&bar_empty[s]), (r - 1) & 1, wc, 11)) return false;
      const int jt = j >> 1;
      int row = (jt < it.nh ? it.hist[jt] * kTile : original_row_kv(d, it.g * d.G + (jt - it.nh) * kTile, it.sh)) +
                (j & 1) * C::BN;
      if (!in_bounds(a.status, row, d.Nk - C::BN + 1, 42)) row = 0;  // debug build: load a valid tile instead
      if (elect_one()) {
        mbar_arrive_expect_tx(smem_u32(&bar_full[s]), C::KV_BYTES);
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(kv_addr(s) + c * C::KV_ATOM, is_v ? &tmV : &tmK, smem_u32(&bar_full[s]), c * 64, it.kvh,
                      row, it.b);
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
        // the next item's first Q tile after this item's first few K/V
        // tiles, this item's second Q tile after its first K/V tile (it goes
        // into the slot the previous item's epilogue releases)
        const int n64 = n_tiles(it, it.has_b ? 1 : 0);
        const int jq = min(5, n64 - 1);
        for (int j = 0; ok && j < n64; ++j) {
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
      for (int s = 0; s < NQ && s < qu; ++s) drain_wait(smem_u32(&bar_qfull[s]), ((qu - 1 - s) / NQ) & 1);
      for (int s = 0; s < NS && s < L; ++s) drain_wait(smem_u32(&bar_full[s]), ((L - 1 - s) / NS) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer
    const uint32_t idS = make_idesc_bf16(128, C::BN, 0, 0);  // Q K-major, K K-major
    const uint32_t idO = make_idesc_bf16(128, D, 0, 1);      // P from TMEM, V MN-major
    const uint64_t dQ0 = make_sdesc_sw128(q_addr(0), 16, 1024);
    const uint64_t dK0 = make_sdesc_sw128(kv_addr(0), 16, 1024);
    const uint64_t dV0 = make_sdesc_sw128(kv_addr(0), C::KV_ATOM, 1024);
    auto commit = [&](uint64_t* bar) {
      if (elect_one()) umma_commit(smem_u32(bar));
      __syncwarp();
    };
    auto wait_full = [&](int Lx) { return warp_wait(smem_u32(&bar_full[Lx % NS]), (Lx / NS) & 1, wc, 20); };
    auto wait_q = [&](int use, uint32_t where) {
      return warp_wait(smem_u32(&bar_qfull[use % NQ]), (use / NQ) & 1, wc, where);
    };
    // an item without a second query tile releases that Q slot here
    auto release_q = [&](int slot) {
      for (int i = 0; i < 4; ++i) commit(&bar_qempty[slot]);
    };
    // S_wg(buffer buf) = Q(slot qs) K(load Lk)^T, 64 keys
    auto issue_s = [&](int wg, int qs, int Lk, int buf) -> bool {
      if (!wait_full(Lk)) return false;
      tc_fence_after();
      const uint64_t dq = sdesc_advance(dQ0, qs * C::Q_BYTES);
      const uint64_t dk = sdesc_advance(dK0, (Lk % NS) * C::KV_BYTES);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_ss(tmem + wg * 128 + buf * 64, sdesc_advance(dq, (kk >> 2) * C::Q_ATOM + (kk & 3) * 32),
                  sdesc_advance(dk, (kk >> 2) * C::KV_ATOM + (kk & 3) * 32), idS, kk > 0);
        umma_commit(smem_u32(&bar_s[wg][buf]));
      }
      __syncwarp();
      return true;
    };
    int L = 0, n = 0, np[2][2] = {{0, 0}, {0, 0}};  // ring loads, items consumed, P tiles received per buffer
    // O_wg (+)= P_wg(j) V(load Lv) once P(j) is in TMEM (and, for an item's
    // first tile, once the epilogue has read the previous item's O)
    auto pv = [&](int wg, int Lv, int j) -> bool {
      if (!warp_wait(smem_u32(&bar_p[wg][j & 1]), np[wg][j & 1] & 1, wc, wg == 0 ? 22 : 24) ||
          (j == 0 && n > 0 && !warp_wait(smem_u32(&bar_ofree[wg]), (n - 1) & 1, wc, wg == 0 ? 23 : 25)) ||
          !wait_full(Lv))
        return false;
      tc_fence_after();
      const uint64_t dv = sdesc_advance(dV0, (Lv % NS) * C::KV_BYTES);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk)
          umma_ts(tmem + C::TM_O + wg * D, tmem + wg * 128 + (j & 1) * 64 + kk * 8, sdesc_advance(dv, kk * 2048),
                  idO, j > 0 || kk > 0);
        umma_commit(smem_u32(&bar_o[wg]));
      }
      __syncwarp();
      ++np[wg][j & 1];
      return true;
    };
    bool pre = false;  // this item's first scores were issued during the previous item
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
      const int nA = n_tiles(it, 0), nB = n_tiles(it, 1), n64 = nA > nB ? nA : nB;
      const int L0 = L;  // K_j is load L0 + 2j, V_j load L0 + 2j + 1
      const int L0n = L0 + 2 * n64;
      if (!pre) {
        if (!wait_q(uA, 21) || !wait_q(uB, 21)) break;
        for (int e = 0; ok && e < 2; ++e) {
          ok = issue_s(0, sA, L0 + 2 * e, e) && (!it.has_b || issue_s(1, sB, L0 + 2 * e, e));
          if (ok && !it.has_b && e == 0) release_q(sB);
          if (ok) commit(&bar_empty[(L0 + 2 * e) % NS]);
        }
        if (!ok) break;
      } else if (!it.has_b) {
        // the absent second tile's Q slot goes back here, once every UMMA of
        // the previous item is issued (any earlier could hold up that item's
        // second-tile work, whose released K/V slots the producer needs first)
        if (!wait_q(uB, 26)) break;
        release_q(sB);
      }
      // the next item's first two scores of warpgroup B (after B's -- or, for
      // an item without B, A's -- last P V of this item)
      auto start_next_b = [&]() -> bool {
        if (!wait_q(uB + 2, 27)) return false;
        for (int e = 0; e < 2; ++e) {
          if (!issue_s(1, sBn, L0n + 2 * e, e)) return false;
          commit(&bar_empty[(L0n + 2 * e) % NS]);
        }
        return true;
      };
      for (int j = 0; ok && j < n64; ++j) {
        const int Lv = L0 + 2 * j + 1;
        if (j < nA) {
          if (!(ok = pv(0, Lv, j))) break;
          if (j >= nB) commit(&bar_empty[Lv % NS]);
          const int t = j + 2;
          if (t < nA) {
            if (!(ok = issue_s(0, sA, L0 + 2 * t, t & 1))) break;
            if (t >= nB) commit(&bar_empty[(L0 + 2 * t) % NS]);
          } else if (nx.valid) {
            const int e = t - nA;
            if (!(ok = wait_q(uA + 2, 26) && issue_s(0, sAn, L0n + 2 * e, e))) break;
            if (!itn.has_b) commit(&bar_empty[(L0n + 2 * e) % NS]);
            if (e == 1 && itn.has_b && !it.has_b && !(ok = start_next_b())) break;  // A's last P V is issued
          }
        }
        if (j < nB) {
          if (!(ok = pv(1, Lv, j))) break;
          commit(&bar_empty[Lv % NS]);
          const int t = j + 2;
          if (t < nB) {
            if (!(ok = issue_s(1, sB, L0 + 2 * t, t & 1))) break;
            commit(&bar_empty[(L0 + 2 * t) % NS]);
          } else if (nx.valid && itn.has_b && t - nB == 1 && !(ok = start_next_b())) {
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
    int nsb[2] = {0, 0};  // uses of each score buffer so far
    int no = 0;           // P tiles handed to the issuer (one P V each)
    int n_item = 0;       // items walked (the Q-ring use of this warpgroup's tile is 2 n_item + wg)
    FwdCursor cur;
    cur.first(a.sched);
    bool ok = true;
    while (ok && cur.valid) {
      const FwdItem it = fwd_item(d, cur.unit, cur.i, a.hist);
      const int t = it.ta + wg;
      const int nt = n_tiles(it, wg);
      if (nt > 0) {
        float m_run = 0.f, l_run = 0.f;
        for (int j = 0; j < nt; ++j) {
          const int buf = j & 1;
          ok = warp_wait(smem_u32(&bar_s[wg][buf]), nsb[buf] & 1, wc, 30);
          if (!ok) break;
          ++nsb[buf];
          tc_fence_after();
          uint32_t sr[2][32];
          tmem_ld32(tS + buf * 64, sr[0]);
          tmem_ld32(tS + buf * 64 + 32, sr[1]);
          tmem_wait_ld();
          if (d.causal && j >= nt - 2) {  // the diagonal 128-key tile: keys after the query are masked
            const int kb = (j - (nt - 2)) * 64;
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (kb + c > row) sr[c >> 5][c & 31] = __float_as_uint(neg_inf());
          }
          float m4[4] = {neg_inf(), neg_inf(), neg_inf(), neg_inf()};
#pragma unroll
          for (int c = 0; c < 64; c += 8) {
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
          // P (bf16) over the first 32 columns of the buffer; every score
          // column of this thread's row was read above
          uint32_t pk[32];
          const float rs = softmax_row64(sr[0], sr[1], sl2, m_run, pk);
          tmem_st32(tS + buf * 64, pk);
          if (__any_sync(0xffffffffu, resc)) {
            // rescale O (it holds P V up to tile j-1 once that UMMA has
            // completed) before P(j) V(j) accumulates onto it.  P V(j-2) is
            // complete (S(j) was issued after it), so only P V(j-1) can be
            // pending and the parity wait is unambiguous
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
          l_run = l_run * alpha + rs;
          if (j == nt - 1) {
            // the item's last P: P V(j-1) completes before P V(j) can be
            // issued, so the epilogue's parity wait below finds one P V phase
            // outstanding, never two (two would leave a parity wait on the
            // earlier one naming a phase the barrier has already passed twice)
            ok = warp_wait(smem_u32(&bar_o[wg]), (no - 1) & 1, wc, 33);
            if (!ok) break;
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&bar_p[wg][buf]));
          ++no;
        }
        // ---------------------------------------------------------- epilogue
        // Only the last P V can still be in flight: P V(nt - 2) was waited
        // for before the last P went out.
        if (ok) ok = warp_wait(smem_u32(&bar_o[wg]), (no - 1) & 1, wc, 32);
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
        // reader (this tile's last S) has completed; one TMA store per
        // 64-column slab; the slot goes back to the producer once read
        const int qs = (2 * n_item + wg) % NQ;
        const uint32_t stage = q_addr(qs) + row * 128;
        const uint32_t sw = static_cast<uint32_t>(row & 7);
#pragma unroll
        for (int sl = 0; sl < D / 64; ++sl) {
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const uint32_t* src = &o[2 * sl + (ch >> 2)][(ch & 3) * 8];
            st_shared_v4(stage + sl * C::Q_ATOM + ((ch ^ sw) << 4),
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
            tma_store_4d(&tmO, q_addr(qs) + sl * C::Q_ATOM + quarter * 32 * 128, sl * 64, it.h, tq0 + quarter * 32,
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
cudaError_t launch_fwd64_slots(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                               const CUtensorMap& to, const FwdArgs& a, int num_sms, cudaStream_t stream) {
  using C = Fwd64Cfg<D, KVS>;
  cudaError_t ea = cudaFuncSetAttribute(s2_fwd64_kernel<D, KVS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        C::SMEM_BYTES);
  if (ea != cudaSuccess) return ea;
  const int grid = a.sched.n < num_sms ? a.sched.n : num_sms;
  prof_before(stream, kKernelFwd);
  s2_fwd64_kernel<D, KVS><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, to, a);
  cudaError_t e = cudaGetLastError();
  prof_after(stream);
  return e;
}

// The 64-key forward: 8 K/V slots of 64 rows at head dim 128, 8 or 12 at 64;
// anything else is an invalid value.  Its K/V tensor maps have 64-row boxes.
template <int D>
cudaError_t launch_fwd64(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& to,
                         const FwdArgs& a, int num_sms, cudaStream_t stream, int kv_slots) {
  if constexpr (D == 128) {
    if (kv_slots == 8) return launch_fwd64_slots<D, 8>(tq, tk, tv, to, a, num_sms, stream);
  } else {
    if (kv_slots == 8) return launch_fwd64_slots<D, 8>(tq, tk, tv, to, a, num_sms, stream);
    if (kv_slots == 12) return launch_fwd64_slots<D, 12>(tq, tk, tv, to, a, num_sms, stream);
  }
  return cudaErrorInvalidValue;
}

template cudaError_t launch_fwd64<64>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                      const CUtensorMap&, const FwdArgs&, int, cudaStream_t, int);
template cudaError_t launch_fwd64<128>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                       const CUtensorMap&, const FwdArgs&, int, cudaStream_t, int);

}  // namespace s2
