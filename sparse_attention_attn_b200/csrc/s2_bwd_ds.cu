// dQ of S2 attention from the dS the dK/dV kernel has already formed
// (backward path "split-dS").  The dK/dV kernel computes dS^T = P^T o (dP^T -
// Delta) for every (kv tile, query sub-tile) pair of a group anyway; on this
// path its elementwise warps also store those bf16 values in the workspace, one
// 128 x 128 block per (query tile i, kv tile j <= i) of each (batch, head,
// group), as four slabs of 32 query columns ([kv][32 queries], 64-byte rows,
// so the dK/dV warps' stores are contiguous).  dQ is then a plain GEMM per
// query tile:
//   dQ_i = scale * sum_{j <= i} dS_ij K_j,
// so the backward issues the five GEMM-units of work the method counts (S^T,
// dP^T, dV, dK in the dK/dV kernel, this one) instead of recomputing S and dP.
// It costs the dS round trip through HBM (B H (N/G) (T (T+1) / 2) 32 KB,
// T = G/128), so the host takes it only while that stays moderate.
//
// Persistent: one CTA per SM walks 128-row query tiles in the pair schedule
// of the other backward kernels (tile t with tile T-1-t: equal work).  Warp 0
// loads, per kv tile j, the dS block (its four slabs with the 64-byte
// swizzle) and K_j (128 rows, D/64 slabs, 128-byte swizzle) into a stage;
// warp 1 issues the SS UMMAs
// (M = 128 query rows, N = D, K = 16 kv rows; A = dS block MN-major, B = K_j
// MN-major) into one of two TMEM accumulators; warps 2-5 (one per TMEM lane
// quarter) scale the finished dQ, stage it as bf16 with the 128-byte swizzle
// and write it with TMA stores at the tile's original (unrolled) rows, while
// the other accumulator takes the next item.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "s2_common.cuh"
#include "s2_ptx.cuh"

namespace s2 {

template <int D, int NST>
struct DqDsCfg {
  static constexpr int STAGES = NST;
  static constexpr int SLAB = kTile * 128;            // K: 128 rows x 64 bf16 columns
  static constexpr int DS_SLAB = kTile * 64;          // dS: 128 rows x 32 bf16 columns
  static constexpr int DS_BYTES = 4 * DS_SLAB;        // one dS block (128 x 128)
  static constexpr int K_BYTES = (D / 64) * SLAB;     // one K tile (128 x D)
  static constexpr int STAGE_BYTES = DS_BYTES + K_BYTES;
  static constexpr int OUT_WARP = 32 * D * 2;         // one epilogue warp's 32 rows of dQ
  static constexpr int OFF_OUT = STAGES * STAGE_BYTES;
  static constexpr int SMEM_BYTES = OFF_OUT + 4 * OUT_WARP + 1024;
  static constexpr int THREADS = 192;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static_assert(2 * D <= 256, "two accumulators in 256 TMEM columns");
};

template <int D, int NST>
__global__ void __launch_bounds__(192, 1)
    s2_bwd_dq_ds_kernel(const __grid_constant__ CUtensorMap tmS, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmQo, const BwdArgs a) {
  using C = DqDsCfg<D, NST>;
  constexpr int ST = C::STAGES;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) uint64_t bar_full[ST], bar_empty[ST], bar_acc_full[2], bar_acc_empty[2], bar_drain;
  __shared__ uint32_t tmem_slot;
  __shared__ uint32_t abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Dims& d = a.d;
  const PairSched& ps = a.q_sched;
  WaitCtx wc{&abort_flag, a.status, a.wait_limit_ns};
  const uint32_t s0 = smem_u32(smem);
  auto sS = [&](int s) { return s0 + s * C::STAGE_BYTES; };
  auto sK = [&](int s) { return s0 + s * C::STAGE_BYTES + C::DS_BYTES; };

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < ST; ++s) {
      mbar_init(smem_u32(&bar_full[s]), 1);
      mbar_init(smem_u32(&bar_empty[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bar_acc_full[i]), 1);
      mbar_init(smem_u32(&bar_acc_empty[i]), 4);  // one arrival per epilogue warp
    }
    mbar_init(smem_u32(&bar_drain), 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_slot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      tma_prefetch_desc(&tmS);
      tma_prefetch_desc(&tmK);
    }
    __syncwarp();
    int L = 0;
    bool ok = true;
    ItemCursor ic;
    for (ic.first(ps); ok && ic.valid; ic.next(ps)) {
      const TileWork w = q_item(d, ic.unit, ic.tile);
      const int sh = shift_of_head(d, w.h);
      const long long blk0 = ds_block(d, w.b, w.h, w.g, w.tile, 0, a.ds_tt, a.ds_slots);
      for (int j = 0; j <= w.tile; ++j, ++L) {
        const int s = L % ST, f = L / ST;
        if (f > 0 && !warp_wait(smem_u32(&bar_empty[s]), (f - 1) & 1, wc, 300)) {
          ok = false;
          break;
        }
        const int tk0 = original_row_kv(d, w.g * d.G + j * kTile, sh);
        const int srow = static_cast<int>((blk0 + j) * 4 * kTile);  // the block's first slab row
        if (elect_one()) {
          const uint32_t bar = smem_u32(&bar_full[s]);
          mbar_arrive_expect_tx(bar, C::STAGE_BYTES);
          tma_load_2d(sS(s), &tmS, bar, 0, srow);                           // slabs 0, 1
          tma_load_2d(sS(s) + 2 * C::DS_SLAB, &tmS, bar, 0, srow + 2 * kTile);  // slabs 2, 3
          for (int c = 0; c < D / 64; ++c) tma_load_4d(sK(s) + c * C::SLAB, &tmK, bar, c * 64, w.kvh, tk0, w.b);
        }
        __syncwarp();
      }
    }
    if (*wc.abort && lane == 0) {
      for (int s = 0; s < ST && s < L; ++s) drain_wait(smem_u32(&bar_full[s]), ((L - 1 - s) / ST) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer
    const uint32_t idQ = make_idesc_bf16(128, D, 1, 1);  // A = dS (query rows contiguous), B = K (MN-major)
    const uint64_t dA0 = make_sdesc_sw64(sS(0), C::DS_SLAB, 512);   // 32-query slabs of 64-byte rows
    const uint64_t dB0 = make_sdesc_sw128(sK(0), C::SLAB, 1024);
    int L = 0, n = 0;
    bool ok = true;
    ItemCursor ic;
    for (ic.first(ps); ok && ic.valid; ic.next(ps), ++n) {
      const TileWork w = q_item(d, ic.unit, ic.tile);
      const int ab = n & 1;
      if (n >= 2 && !warp_wait(smem_u32(&bar_acc_empty[ab]), ((n >> 1) - 1) & 1, wc, 301)) break;
      tc_fence_after();
      for (int j = 0; j <= w.tile; ++j, ++L) {
        const int s = L % ST;
        if (!warp_wait(smem_u32(&bar_full[s]), (L / ST) & 1, wc, 302)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
          const uint64_t da = sdesc_advance(dA0, s * C::STAGE_BYTES);
          const uint64_t db = sdesc_advance(dB0, s * C::STAGE_BYTES);
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            umma_ss(tmem + ab * D, sdesc_advance(da, kk * 1024), sdesc_advance(db, kk * 2048), idQ,
                    (j > 0 || kk > 0));
          umma_commit(smem_u32(&bar_empty[s]));
          if (j == w.tile) umma_commit(smem_u32(&bar_acc_full[ab]));
        }
        __syncwarp();
      }
    }
    if (elect_one()) {
      umma_commit(smem_u32(&bar_drain));
      drain_wait(smem_u32(&bar_drain), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t stage = s0 + C::OFF_OUT + quarter * C::OUT_WARP;
    int n = 0;
    ItemCursor ic;
    for (ic.first(ps); ic.valid; ic.next(ps), ++n) {
      const TileWork w = q_item(d, ic.unit, ic.tile);
      const int ab = n & 1;
      const int tq0 = original_row(d, w.g * d.G + w.tile * kTile, shift_of_head(d, w.h));
      if (!warp_wait(smem_u32(&bar_acc_full[ab]), (n >> 1) & 1, wc, 303)) break;
      // the previous store has finished reading the staging rows
      if (lane == 0) bulk_wait_read_all();
      __syncwarp();
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_off + ab * D + c * 32, r);
        tmem_wait_ld();
        // 32 columns = 4 chunks of 16 bytes in slab c / 2, chunks 4 (c & 1) + q
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int ch = 4 * (c & 1) + q;
          st_shared_v4(stage + (c >> 1) * (32 * 128) + lane * 128 + ((ch ^ (lane & 7)) << 4),
                       pack_bf16x2(__uint_as_float(r[8 * q]) * a.scale, __uint_as_float(r[8 * q + 1]) * a.scale),
                       pack_bf16x2(__uint_as_float(r[8 * q + 2]) * a.scale, __uint_as_float(r[8 * q + 3]) * a.scale),
                       pack_bf16x2(__uint_as_float(r[8 * q + 4]) * a.scale, __uint_as_float(r[8 * q + 5]) * a.scale),
                       pack_bf16x2(__uint_as_float(r[8 * q + 6]) * a.scale, __uint_as_float(r[8 * q + 7]) * a.scale));
        }
      }
      // dQ is out of TMEM: the accumulator takes the item after next
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(&bar_acc_empty[ab]));
        for (int sl = 0; sl < D / 64; ++sl)
          tma_store_4d(&tmQo, stage + sl * (32 * 128), sl * 64, w.h, tq0 + quarter * 32, w.b);
        bulk_commit_group();
      }
      __syncwarp();
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <int D, int NST>
cudaError_t launch_dq_ds_stages(const CUtensorMap& tds, const CUtensorMap& tk, const CUtensorMap& tq32,
                                const BwdArgs& a, int num_sms, cudaStream_t stream) {
  using C = DqDsCfg<D, NST>;
  cudaError_t ea =
      cudaFuncSetAttribute(s2_bwd_dq_ds_kernel<D, NST>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (ea != cudaSuccess) return ea;
  const int grid = pair_grid(a.q_sched, num_sms);
  prof_before(stream, kKernelBwdDqDs);
  s2_bwd_dq_ds_kernel<D, NST><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tds, tk, tq32, a);
  cudaError_t e = cudaGetLastError();
  prof_after(stream);
  return e;
}

// The dQ-from-dS kernel: 3 stages of (dS block, K tile) at head dim 128, 4 at 64.
template <int D>
cudaError_t launch_dq_ds(const CUtensorMap& tds, const CUtensorMap& tk, const CUtensorMap& tq32, const BwdArgs& a,
                         int num_sms, cudaStream_t stream) {
  if constexpr (D == 128)
    return launch_dq_ds_stages<D, 3>(tds, tk, tq32, a, num_sms, stream);
  else
    return launch_dq_ds_stages<D, 4>(tds, tk, tq32, a, num_sms, stream);
}

template cudaError_t launch_dq_ds<64>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const BwdArgs&,
                                      int, cudaStream_t);
template cudaError_t launch_dq_ds<128>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                       const BwdArgs&, int, cudaStream_t);

}  // namespace s2
