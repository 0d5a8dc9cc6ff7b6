// dK / dV of S2-Attn with 128-query tiles, for sm_100a.
//
// The same work as the dK/dV kernel in s2_bwd.cu (per 128-row kv tile of one
// rolled group of one (batch, kv head): dV = sum P^T dO, dK = scale sum dS^T Q
// over the query tiles from the diagonal to the group end and the query heads
// that share the kv head -- LongQLoRA community post, section 03; the analytic
// backward of softmax attention), with the query side in 128-row tiles
// instead of 64-row sub-tiles.  S^T = K Q^T and dP^T = V dO^T are then UMMAs
// with N = 128: twice the work per instruction, and balanced between the
// tensor pipe and shared-memory bandwidth (an N = 64 SS UMMA reads 6 KB of
// operands per 16-deep step for 128 x 64 outputs), so the two issuing threads
// keep the pipe fed with a third fewer instructions.
//
// TMEM holds S^T and dP^T of one query tile (128 columns each) beside the dV
// and dK accumulators (D columns each): one buffer, so each query tile is
// worked in two 64-query halves.  The elementwise warps turn the first half
// of S^T / dP^T into P^T / dS^T and release it; the issuers start dV / dK on
// it while the second half is being formed; the next tile's S^T / dP^T follow
// the second half's gradient UMMAs in each issuer's stream, so they never
// overwrite a value that is still to be read.
//
// Warps: 0 TMA producer (K/V of the item, then 128-row Q / dO tiles and their
// row statistics through a ring), 1 issuer A (TMEM owner; S^T and dV),
// 2..9 elementwise and epilogue (warp w: TMEM lanes 32 (w mod 4) .. +31 = its
// kv rows, 32-column halves (w - 2) / 4 of each 64-query half), 10 issuer B
// (dP^T and dK).  TMEM: S^T [0,128), dP^T [128,256), dV [256, 256+D),
// dK [256+D, 256+2D); P^T / dS^T are written as bf16 pairs over the first 16
// of each warp's 32 columns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "s2_common.cuh"
#include "s2_ptx.cuh"

namespace s2 {

template <int D, int NST>
struct Kv128Cfg {
  static constexpr int STAGES = NST;
  static constexpr int ATOM = kTile * 128;      // one 64-column slab of a 128-row tile
  static constexpr int TILE_BYTES = kTile * D * 2;
  static constexpr int OFF_KV = 0;              // [K, V] of the current item
  static constexpr int OFF_Q = 2 * TILE_BYTES;  // per stage: Q tile, dO tile
  static constexpr int OFF_ROW = OFF_Q + STAGES * 2 * TILE_BYTES;  // per stage: -lse2[128], -delta[128]
  static constexpr int SMEM_BYTES = OFF_ROW + STAGES * 1024 + 1024;
  static_assert(SMEM_BYTES <= 232448 - 512, "shared memory");
  static constexpr uint32_t TM_S = 0, TM_DP = 128, TM_DV = 256, TM_DK = 256 + D;
  static constexpr int THREADS = 352;
};

// Query-tile cursor of one CTA: item (kv tile) and query-tile index inside it
// (query head it / nq, query tile w.tile + it % nq of the group).
struct Kv128Cursor {
  ItemCursor ic;
  TileWork w;
  int it, iters, nq;
  __device__ __forceinline__ void load(const Dims& d) {
    if (!ic.valid) return;
    w = kv_item(d, ic.unit, ic.tile);
    nq = d.tiles - w.tile;
    iters = d.rep * nq;
    it = 0;
  }
  __device__ __forceinline__ void first(const Dims& d, const PairSched& ps) {
    ic.first(ps);
    load(d);
  }
  __device__ __forceinline__ void next(const Dims& d, const PairSched& ps) {
    if (++it < iters) return;
    ic.next(ps);
    load(d);
  }
};

template <int D, int NST>
__global__ void __launch_bounds__(352, 1)
    s2_bwd_dkdv128_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmG,
                          const BwdArgs a) {
  using C = Kv128Cfg<D, NST>;
  constexpr int ST = C::STAGES;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  // kv / kv_empty: the item's K/V landed / released (after its last S^T and
  // dP^T, one commit per issuer); full / empty: a query stage landed /
  // released (after both issuers' last gradient UMMAs on it); s / dp: S^T /
  // dP^T of a query tile landed; p[h]: half h of P^T / dS^T written (one
  // arrival per elementwise warp); acc_full / acc_free: the item's dV / dK
  // complete / read out.
  __shared__ __align__(8) uint64_t bar_kv, bar_kv_empty, bar_full[ST], bar_empty[ST], bar_s, bar_dp, bar_p[2],
      bar_acc_full, bar_acc_free, bar_drain[2];
  __shared__ uint32_t tmem_slot;
  __shared__ uint32_t abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Dims& d = a.d;
  const PairSched& ps = a.kv_sched;
  WaitCtx wc{&abort_flag, a.status, a.wait_limit_ns};

  const uint32_t s0 = smem_u32(smem);
  const uint32_t sK = s0 + C::OFF_KV, sV = s0 + C::OFF_KV + C::TILE_BYTES;
  auto sQ = [&](int s) { return s0 + C::OFF_Q + s * 2 * C::TILE_BYTES; };
  auto sG = [&](int s) { return s0 + C::OFF_Q + s * 2 * C::TILE_BYTES + C::TILE_BYTES; };
  auto sRow = [&](int s) { return s0 + C::OFF_ROW + s * 1024; };

  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar_kv), 1);
    mbar_init(smem_u32(&bar_kv_empty), 2);
    for (int s = 0; s < ST; ++s) {
      mbar_init(smem_u32(&bar_full[s]), 1);
      mbar_init(smem_u32(&bar_empty[s]), 2);
    }
    mbar_init(smem_u32(&bar_s), 1);
    mbar_init(smem_u32(&bar_dp), 1);
    for (int h = 0; h < 2; ++h) {
      mbar_init(smem_u32(&bar_p[h]), 8);
      mbar_init(smem_u32(&bar_drain[h]), 1);
    }
    mbar_init(smem_u32(&bar_acc_full), 2);
    mbar_init(smem_u32(&bar_acc_free), 8);
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
      tma_prefetch_desc(&tmG);
    }
    __syncwarp();
    int gi = 0, kv_issued = 0;
    bool ok = true;
    ItemCursor ic;
    for (ic.first(ps); ok && ic.valid; ic.next(ps)) {
      const TileWork w = kv_item(d, ic.unit, ic.tile);
      const int sh = shift_of_head(d, w.h);
      if (ic.n >= 1 && !warp_wait(smem_u32(&bar_kv_empty), (ic.n - 1) & 1, wc, 150)) break;
      const int tk0 = original_row_kv(d, d.qoff_t * kTile + w.g * d.G + w.tile * kTile, sh);
      if (elect_one()) {
        mbar_arrive_expect_tx(smem_u32(&bar_kv), 2 * C::TILE_BYTES);
        for (int c = 0; c < D / 64; ++c) {
          tma_load_4d(sK + c * C::ATOM, &tmK, smem_u32(&bar_kv), c * 64, w.kvh, tk0, w.b);
          tma_load_4d(sV + c * C::ATOM, &tmV, smem_u32(&bar_kv), c * 64, w.kvh, tk0, w.b);
        }
      }
      __syncwarp();
      ++kv_issued;
      const int nq = d.tiles - w.tile;
      const int iters = d.rep * nq;
      for (int it = 0; it < iters; ++it, ++gi) {
        const int s = gi % ST, f = gi / ST;
        if (f > 0 && !warp_wait(smem_u32(&bar_empty[s]), (f - 1) & 1, wc, 151)) {
          ok = false;
          break;
        }
        const int h = w.kvh * d.rep + it / nq;
        const int tq0 = original_row(d, w.g * d.G + (w.tile + it % nq) * kTile, sh);
        const uint32_t bar = smem_u32(&bar_full[s]);
        if (elect_one()) {
          mbar_arrive_expect_tx(bar, 2 * C::TILE_BYTES + 1024);
          for (int c = 0; c < D / 64; ++c) {
            tma_load_4d(sQ(s) + c * C::ATOM, &tmQ, bar, c * 64, h, tq0, w.b);
            tma_load_4d(sG(s) + c * C::ATOM, &tmG, bar, c * 64, h, tq0, w.b);
          }
          const size_t ro = (static_cast<size_t>(w.b) * d.H + h) * d.N + tq0;
          bulk_load(sRow(s), a.nlse2 + ro, 512, bar);
          bulk_load(sRow(s) + 512, a.ndelta + ro, 512, bar);
        }
        __syncwarp();
      }
    }
    if (*wc.abort && lane == 0) {
      // never leave copies in flight into shared memory
      if (kv_issued > 0) drain_wait(smem_u32(&bar_kv), (kv_issued - 1) & 1);
      for (int s = 0; s < ST && s < gi; ++s) drain_wait(smem_u32(&bar_full[s]), ((gi - 1 - s) / ST) & 1);
    }
  } else if (warp == 1 || warp == 10) {
    // ------------------------------------------------------------ UMMA issuers
    // A (warp 1): S^T = K Q^T, dV += P^T dO.  B (warp 10): dP^T = V dO^T,
    // dK += dS^T Q.  Per query tile: the scores, then the gradient UMMAs of
    // each 64-query half once the elementwise warps have released it.
    const bool A = (warp == 1);
    const uint32_t idS = make_idesc_bf16(128, kTile, 0, 0);  // S^T, dP^T: M = kv rows, N = 128 queries
    const uint32_t idG = make_idesc_bf16(128, D, 0, 1);      // dV, dK: N = D, B MN-major
    const uint64_t dX0 = make_sdesc_sw128(A ? sK : sV, 16, 1024);                 // K-major (A operand)
    const uint64_t dYk = make_sdesc_sw128(A ? sQ(0) : sG(0), 16, 1024);           // K-major (B of S^T / dP^T)
    const uint64_t dZm = make_sdesc_sw128(A ? sG(0) : sQ(0), C::ATOM, 1024);      // MN-major (B of dV / dK)
    const uint32_t tm_sp = tmem + (A ? C::TM_S : C::TM_DP);
    const uint32_t tm_acc = tmem + (A ? C::TM_DV : C::TM_DK);
    const uint32_t bar_ready = smem_u32(A ? &bar_s : &bar_dp);
    Kv128Cursor cur;
    cur.first(d, ps);
    bool ok = true;
    for (int g = 0; ok && cur.ic.valid; ++g) {
      const int s = g % ST;
      if (cur.it == 0 && !warp_wait(smem_u32(&bar_kv), cur.ic.n & 1, wc, 160)) break;
      if (!warp_wait(smem_u32(&bar_full[s]), (g / ST) & 1, wc, 161)) break;
      tc_fence_after();
      const bool last = (cur.it == cur.iters - 1);
      const uint64_t dy = sdesc_advance(dYk, s * 2 * C::TILE_BYTES);
      if (elect_one()) {
        // S^T (dP^T) of this query tile: its TMEM region's last readers (the
        // previous tile's gradient UMMAs of this issuer) were issued before
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::ATOM + (kk & 3) * 32;
          umma_ss(tm_sp, sdesc_advance(dX0, off), sdesc_advance(dy, off), idS, kk > 0);
        }
        umma_commit(bar_ready);
        if (last) umma_commit(smem_u32(&bar_kv_empty));
      }
      __syncwarp();
      const uint64_t dz = sdesc_advance(dZm, s * 2 * C::TILE_BYTES);
      for (int h = 0; h < 2; ++h) {
        if (!warp_wait(smem_u32(&bar_p[h]), g & 1, wc, 162 + h)) {
          ok = false;
          break;
        }
        if (h == 0 && cur.it == 0 && cur.ic.n > 0 &&
            !warp_wait(smem_u32(&bar_acc_free), (cur.ic.n - 1) & 1, wc, 164)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
          // K-step kk of this half: queries 64 h + 16 kk .. +15, written (as
          // bf16 pairs) by the warps of column half kk / 2 at packed columns
          // 64 h + 32 (kk / 2) + 8 (kk mod 2)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_ts(tm_acc, tm_sp + 64 * h + 32 * (kk >> 1) + 8 * (kk & 1),
                    sdesc_advance(dz, (4 * h + kk) * 2048), idG, (cur.it > 0 || h > 0 || kk > 0));
          if (h == 1) {
            umma_commit(smem_u32(&bar_empty[s]));
            if (last) umma_commit(smem_u32(&bar_acc_full));
          }
        }
        __syncwarp();
      }
      cur.next(d, ps);
    }
    if (elect_one()) {
      umma_commit(smem_u32(&bar_drain[A ? 0 : 1]));
      drain_wait(smem_u32(&bar_drain[A ? 0 : 1]), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ P^T, dS^T, epilogue
    const int quarter = warp & 3;
    const int col = (warp - 2) >> 2;      // 32-column half of each 64-query half
    const int row = quarter * 32 + lane;  // kv row inside the tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float sl2 = a.scale_log2;
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    bool ok = true;
    Kv128Cursor cur;
    cur.first(d, ps);
    long long ds_base = 0;
    for (int g = 0; cur.ic.valid; ++g) {
      const int s = g % ST;
      const bool diag = (cur.it % cur.nq) == 0;  // the query tile on the kv tile's diagonal
      ok = warp_wait(smem_u32(&bar_full[s]), (g / ST) & 1, wc, 170) &&
           warp_wait(smem_u32(&bar_s), g & 1, wc, 171) && warp_wait(smem_u32(&bar_dp), g & 1, wc, 172);
      if (!ok) break;
      tc_fence_after();
      if (a.ds != nullptr && cur.it == 0)
        ds_base = ds_block(d, cur.w.b, cur.w.h, cur.w.g, 0, 0, a.ds_tt, a.ds_slots);
      for (int h = 0; h < 2; ++h) {
        const int q0 = 64 * h + 32 * col;  // this warp's first query column of the tile
        const uint32_t l4 = sRow(s) + q0 * 4, d4 = l4 + 512;
        float4 lv[8], dv4[8];
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          lv[c4] = lds_f4(l4 + c4 * 16);
          dv4[c4] = lds_f4(d4 + c4 * 16);
        }
        uint32_t sr[32], dr[32];
        tmem_ld32(tmem + lane_off + C::TM_S + q0, sr);
        tmem_ld32(tmem + lane_off + C::TM_DP + q0, dr);
        tmem_wait_ld();
        float p[32];
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {  // P^T = 2^(S^T * scale * log2 e - lse * log2 e)
          const float4 l = lv[c4];
          const uint64_t x01 = f2_fma(f2_pack(__uint_as_float(sr[4 * c4]), __uint_as_float(sr[4 * c4 + 1])),
                                      sl2x2, f2_pack(l.x, l.y));
          const uint64_t x23 = f2_fma(f2_pack(__uint_as_float(sr[4 * c4 + 2]), __uint_as_float(sr[4 * c4 + 3])),
                                      sl2x2, f2_pack(l.z, l.w));
          p[4 * c4 + 0] = ex2_approx(f2_lo(x01));
          p[4 * c4 + 1] = ex2_approx(f2_hi(x01));
          p[4 * c4 + 2] = ex2_approx(f2_lo(x23));
          p[4 * c4 + 3] = ex2_approx(f2_hi(x23));
        }
        if (diag) {  // diagonal tile: a query before the key is masked
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (q0 + c < row) p[c] = 0.f;
        }
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) pk[c] = pack_bf16x2(p[2 * c], p[2 * c + 1]);
        tmem_st16(tmem + lane_off + C::TM_S + q0, pk);
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {  // dS^T = P^T * (dP^T - Delta)
          const float4 dl = dv4[c4];
          const uint64_t d01 = f2_add(f2_pack(__uint_as_float(dr[4 * c4]), __uint_as_float(dr[4 * c4 + 1])),
                                      f2_pack(dl.x, dl.y));
          const uint64_t d23 = f2_add(f2_pack(__uint_as_float(dr[4 * c4 + 2]), __uint_as_float(dr[4 * c4 + 3])),
                                      f2_pack(dl.z, dl.w));
          dk[2 * c4] = f2_to_bf16x2(f2_mul(f2_pack(p[4 * c4], p[4 * c4 + 1]), d01));
          dk[2 * c4 + 1] = f2_to_bf16x2(f2_mul(f2_pack(p[4 * c4 + 2], p[4 * c4 + 3]), d23));
        }
        tmem_st16(tmem + lane_off + C::TM_DP + q0, dk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bar_p[h]));
        if (a.ds != nullptr) {
          // split-dS path: the query tile is the dS block (i, j) of query
          // tile i = tile + it mod nq and kv tile j = tile, of query head
          // kvh rep + it / nq; these 32 values go to row `row` of its
          // 32-column slab 2 h + col: the warp's 32 rows write 2 KB of
          // consecutive bytes.  After the arrival, so the gradient UMMAs
          // never wait for them.
          const int i = cur.w.tile + cur.it % cur.nq;
          const long long blk =
              ds_base + static_cast<long long>(cur.it / cur.nq) * a.ds_tt + i * (i + 1) / 2 + cur.w.tile;
          if (in_bounds(wc.status, blk, a.ds_blocks, 49)) {
            __nv_bfloat16* dst = a.ds + blk * (kTile * kTile) + (2 * h + col) * (kTile * 32) + row * 32;
            const uint32_t lo[8] = {dk[0], dk[1], dk[2], dk[3], dk[4], dk[5], dk[6], dk[7]};
            const uint32_t hi[8] = {dk[8], dk[9], dk[10], dk[11], dk[12], dk[13], dk[14], dk[15]};
            st_global_v8(dst, lo);
            st_global_v8(dst + 16, hi);
          }
        }
      }
      if (cur.it == cur.iters - 1) {
        // ---------------------------------------------------- epilogue of this item
        ok = warp_wait(smem_u32(&bar_acc_full), cur.ic.n & 1, wc, 173);
        if (!ok) break;
        tc_fence_after();
        const TileWork& w = cur.w;
        const int tk0 = original_row(d, w.g * d.G + w.tile * kTile, shift_of_head(d, w.h));
        const size_t grow = (static_cast<size_t>(w.b) * d.N + tk0 + row) * d.Hkv + w.kvh;
        const bool grow_ok =
            in_bounds(wc.status, static_cast<long long>(grow), static_cast<long long>(d.B) * d.N * d.Hkv, 47);
        __nv_bfloat16* dvrow = static_cast<__nv_bfloat16*>(a.dv) + grow * D + col * (D / 2);
        __nv_bfloat16* dkrow = static_cast<__nv_bfloat16*>(a.dk) + grow * D + col * (D / 2);
        uint32_t r[D / 64][32], r2[D / 64][32];
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          tmem_ld32(tmem + lane_off + C::TM_DV + col * (D / 2) + c * 32, r[c]);
          tmem_ld32(tmem + lane_off + C::TM_DK + col * (D / 2) + c * 32, r2[c]);
        }
        tmem_wait_ld();
        // dV / dK are out of TMEM: the next item's first gradient UMMAs may start
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bar_acc_free));
#pragma unroll
        for (int c = 0; c < D / 64 && grow_ok; ++c) {
          if (a.kv_v8) {
            store_row32_v8(dvrow + c * 32, r[c], 1.f);
            store_row32_v8(dkrow + c * 32, r2[c], a.scale);
          } else {
            store_row32(dvrow + c * 32, r[c], 1.f);
            store_row32(dkrow + c * 32, r2[c], a.scale);
          }
        }
      }
      cur.next(d, ps);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// One launch over a.kv_sched's pair range; stages of 2 x 128-row Q / dO
// tiles: 2 at head dim 128 (what fits beside K and V), 3 at head dim 64.
template <int D>
cudaError_t launch_dkdv128(const BwdMaps& m, const BwdArgs& a, int num_sms, cudaStream_t stream) {
  constexpr int NST = D == 128 ? 2 : 3;
  using C = Kv128Cfg<D, NST>;
  cudaError_t ea = cudaFuncSetAttribute(s2_bwd_dkdv128_kernel<D, NST>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        C::SMEM_BYTES);
  if (ea != cudaSuccess) return ea;
  prof_before(stream, kKernelBwdDkDv);
  s2_bwd_dkdv128_kernel<D, NST><<<pair_grid(a.kv_sched, num_sms), C::THREADS, C::SMEM_BYTES, stream>>>(
      m.q128, m.k128, m.v128, m.g128, a);
  cudaError_t e = cudaGetLastError();
  prof_after(stream);
  return e;
}

template cudaError_t launch_dkdv128<64>(const BwdMaps&, const BwdArgs&, int, cudaStream_t);
template cudaError_t launch_dkdv128<128>(const BwdMaps&, const BwdArgs&, int, cudaStream_t);

}  // namespace s2
