// QKV projection from 4-bit NormalFloat weights with double quantization
// (LongQLoRA community post, section 03 Method, QLoRA: the frozen weights are
// held in 4-bit NF4 and their quantization constants quantized once more;
// section 04: the whole model is quantized this way, so the q, k and v that
// S2 attention takes come out of these projections).
//
// Weight layout (W is [Nout, K], Nout = (H + 2 Hkv) D rows = output features,
// K = model width; row n of W produces feature n):
//   codes  uint8 [Nout, K/2]: element 2j of a row in the low nibble of byte j,
//          element 2j+1 in the high nibble;
//   sq     int8  [Nout * K/64]: first-level scale code of block (n, kb), the 64
//          elements [64 kb, 64 kb + 64) of row n, at n * K/64 + kb;
//   c2     fp32  [ceil(Nout * K/64 / 256)]: second-level scale of every 256
//          consecutive first-level blocks;
//   W'[n, k] = bf16( level[code] * s ),  s = sq * c2 / 127 (fp32 arithmetic),
//   with level[] the 16 NF4 values (host-computed, passed in).
//
// s2_nf4_qkv_kernel computes [q | k | v] = x W'^T on the tensor cores with the
// dequantization fused in: W' never exists in global memory.  The UMMA runs
// with the weight as its A operand held in TMEM: M = 128 weight rows, N = 256
// tokens, K = 16.  Dequantization warps, one per TMEM lane quarter, turn
// each 64-element block of their row into 32 packed bf16 pairs and write them
// straight into a TMEM stage with tcgen05.st, so the dequantized operand costs
// no shared-memory traffic; x comes in by TMA (128-byte swizzle, K-major B
// operand) together with the 4 KB of codes of the stage.  The NF4 lookup is a
// warp shuffle from a 16-entry table held one entry per lane.  Every block of
// 64 elements is one first-level quantization block, so each thread forms one
// scale per stage.
//
// Warp roles (448 threads, one CTA per SM, persistent over the tiles):
//   0      producer: TMA of x [256 tokens x 64] and codes [128 rows x 32 B]
//   1      UMMA issuer (one elected lane)
//   2-9    dequantization into the TMEM A stages, two groups of four taking
//          alternate stages
//   10-13  epilogue: TMEM -> bf16 staging in shared memory -> TMA store to q / k / v
// TMEM: accumulator columns [0, 256), A stages [256 + 32 s, 256 + 32 s + 32).
// Five stages by default: the x tiles come from L2 at about 12 TB/s over all
// SMs, and with four the issuer measurably waited for them.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "s2_common.cuh"
#include "s2_ptx.cuh"

namespace s2 {

// Entry (lane mod 16) of the level table, picked by a select tree on the lane
// bits with static indices only (a dynamic index into the kernel parameters
// would copy them to local memory).
__device__ __forceinline__ float lane_level(const Nf4Levels& lv, int lane) {
  float t[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) t[i] = (lane & 8) ? lv.v[8 + i] : lv.v[i];
#pragma unroll
  for (int i = 0; i < 4; ++i) t[i] = (lane & 4) ? t[4 + i] : t[i];
#pragma unroll
  for (int i = 0; i < 2; ++i) t[i] = (lane & 2) ? t[2 + i] : t[i];
  return (lane & 1) ? t[1] : t[0];
}

template <int NS, int DQW>
struct Nf4Cfg {
  static constexpr int BW = 128, BT = 256, BK = 64;
  static constexpr int X_BYTES = BT * BK * 2;  // 32 KB per stage
  static constexpr int C_BYTES = BW * BK / 2;  // 4 KB per stage
  static constexpr int O_WARP_BYTES = 128 * 32 * 2;  // one epilogue warp's staging: 8 KB (half a tile)
  static constexpr int SMEM_BYTES = NS * (X_BYTES + C_BYTES) + 4 * O_WARP_BYTES + 1024;
  static constexpr int TM_A = 256;
  static constexpr int DQ_WARPS = DQW;  // dequantization warps: groups of four
  static constexpr int THREADS = 32 * (2 + DQ_WARPS + 4);
  static_assert(DQW % 4 == 0 && DQW >= 4, "whole groups of four dequantization warps");
  static_assert(TM_A + 32 * NS <= 512, "A stages must fit in TMEM beside the accumulator");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

template <int NS, int DQW>
__global__ void __launch_bounds__(Nf4Cfg<NS, DQW>::THREADS, 1)
    s2_nf4_qkv_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmC,
                      const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const Nf4Args a) {
  using C = Nf4Cfg<NS, DQW>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) uint64_t bar_full[NS], bar_afull[NS], bar_empty[NS], bar_acc_full, bar_acc_empty,
      bar_drain;
  __shared__ uint32_t tmem_slot;
  __shared__ uint32_t abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  WaitCtx wc{&abort_flag, a.status, a.wait_limit_ns};
  const uint32_t sX = smem_u32(smem), sC = sX + NS * C::X_BYTES, sO = sC + NS * C::C_BYTES;
  const int KB = a.K / 64;
  const int ntiles = a.tiles_w * a.tiles_t;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int s = 0; s < NS; ++s) {
      mbar_init(smem_u32(&bar_full[s]), 1);
      mbar_init(smem_u32(&bar_afull[s]), 4);  // one arrival per warp of the stage's dequantization group
      mbar_init(smem_u32(&bar_empty[s]), 1);
    }
    mbar_init(smem_u32(&bar_acc_full), 1);
    mbar_init(smem_u32(&bar_acc_empty), 4);  // one arrival per epilogue warp
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
      tma_prefetch_desc(&tmX);
      tma_prefetch_desc(&tmC);
    }
    __syncwarp();
    int L = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x) {
      const int tw = tile % a.tiles_w, tt = tile / a.tiles_w;
      for (int kb = 0; kb < KB; ++kb) {
        const int s = L % NS, r = L / NS;
        if (r > 0 && !warp_wait(smem_u32(&bar_empty[s]), (r - 1) & 1, wc, 60)) {
          ok = false;
          break;
        }
        if (elect_one()) {
          const uint32_t bar = smem_u32(&bar_full[s]);
          mbar_arrive_expect_tx(bar, C::X_BYTES + C::C_BYTES);
          tma_load_2d(sX + s * C::X_BYTES, &tmX, bar, kb * 64, tt * C::BT);
          tma_load_2d(sC + s * C::C_BYTES, &tmC, bar, kb * 32, tw * C::BW);
        }
        __syncwarp();
        ++L;
      }
    }
    if (*wc.abort && lane == 0) {
      for (int s = 0; s < NS && s < L; ++s) drain_wait(smem_u32(&bar_full[s]), ((L - 1 - s) / NS) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer
    const uint32_t idesc = make_idesc_bf16(128, C::BT, 0, 0);  // A (weights) from TMEM, x K-major
    const uint64_t dX0 = make_sdesc_sw128(sX, 16, 1024);
    int L = 0, n = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++n) {
      if (n > 0 && !warp_wait(smem_u32(&bar_acc_empty), (n - 1) & 1, wc, 61)) break;
      tc_fence_after();
      for (int kb = 0; kb < KB; ++kb) {
        const int s = L % NS;
        const uint32_t ph = (L / NS) & 1;
        if (!warp_wait(smem_u32(&bar_full[s]), ph, wc, 62) || !warp_wait(smem_u32(&bar_afull[s]), ph, wc, 63)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
          const uint64_t dx = sdesc_advance(dX0, s * C::X_BYTES);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_ts(tmem, tmem + C::TM_A + s * 32 + kk * 8, sdesc_advance(dx, kk * 32), idesc, (kb | kk) != 0);
          umma_commit(smem_u32(&bar_empty[s]));
        }
        __syncwarp();
        ++L;
      }
      if (!ok) break;
      if (elect_one()) umma_commit(smem_u32(&bar_acc_full));
      __syncwarp();
    }
    // every UMMA issued has completed before TMEM is released
    if (elect_one()) {
      umma_commit(smem_u32(&bar_drain));
      drain_wait(smem_u32(&bar_drain), 0);
    }
    __syncwarp();
  } else if (warp < 2 + C::DQ_WARPS) {
    // ------------------------------------------------------------ dequantization
    // DQ_GROUPS groups of four warps take the stages in turn (group g the
    // stages L = g, g + DQ_GROUPS, ...), so one group's shuffles and TMEM
    // store overlap the others'; within a group warp w serves TMEM lanes
    // 32 (w mod 4) + [0, 32).
    constexpr int NG = C::DQ_WARPS / 4;
    const int sub = warp & 3, row = 32 * sub + lane, grp = (warp - 2) >> 2;
    const float table = lane_level(a.lv, lane);
    const uint32_t tA = tmem + (static_cast<uint32_t>(32 * sub) << 16) + C::TM_A;
    auto advance = [&](int& t, int& k) {
      if (++k == KB) {
        k = 0;
        t += gridDim.x;
      }
    };
    // scale code and second-level scale of (tile, kb) for this thread's row,
    // fetched one own stage ahead of their use
    auto fetch = [&](int t, int k, int& q, float& c) {
      const long long blk = static_cast<long long>((t % a.tiles_w) * C::BW + row) * KB + k;
      q = 0;
      c = 0.f;
      if (in_bounds(a.status, blk, static_cast<long long>(a.tiles_w) * C::BW * KB, 47)) {
        q = a.sq[blk];
        c = __ldg(a.c2 + (blk >> 8));
      }
    };
    int tile = blockIdx.x, kb = 0, L = grp;
    for (int i = 0; i < grp; ++i) advance(tile, kb);
    int qn = 0;
    float cn = 0.f;
    if (tile < ntiles) fetch(tile, kb, qn, cn);
    while (tile < ntiles) {
      const int q = qn;
      const float c2 = cn;
      int ntile = tile, nkb = kb;
#pragma unroll
      for (int i = 0; i < NG; ++i) advance(ntile, nkb);
      if (ntile < ntiles) fetch(ntile, nkb, qn, cn);
      const float sc = static_cast<float>(q) * c2 / 127.f;
      const uint64_t sc2 = f2_pack(sc, sc);
      const int s = L % NS;
      // The groups take a stage's loads in turn, so this group skips phases of
      // bar_full[s]: before its parity wait, the stage's previous load must be
      // known to have landed, or a barrier still a phase behind would show the
      // parity of a completed phase and the wait would pass at once.  The
      // UMMA of that load completing (bar_empty[s]) says so, and costs
      // nothing in the normal order: the producer waited for it before it
      // issued this load.
      if (L >= NS && !warp_wait(smem_u32(&bar_empty[s]), (L / NS - 1) & 1, wc, 66)) break;
      if (!warp_wait(smem_u32(&bar_full[s]), (L / NS) & 1, wc, 64)) break;
      const uint32_t src = sC + s * C::C_BYTES + row * 32;
      const uint4 c0 = lds_u4(src), c1 = lds_u4(src + 16);
      const uint32_t wd[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      uint32_t pk[32];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const float lo = warp_lut16(table, wd[i] >> (8 * p));
          const float hi = warp_lut16(table, wd[i] >> (8 * p + 4));
          pk[4 * i + p] = f2_to_bf16x2(f2_mul(f2_pack(lo, hi), sc2));
        }
      }
      tmem_st32(tA + s * 32, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar_afull[s]));
      L += NG;
      tile = ntile;
      kb = nkb;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Each warp owns 32 features of the tile.  Per half of 128 tokens it
    // loads their values from TMEM into registers (bf16 pairs of tokens 2i,
    // 2i + 1), writes them to its [128 tokens][32 features] bf16 staging area
    // (64-byte rows) and stores the area with one TMA copy (rows past M are
    // clipped by the copy).  The accumulator is released as soon as the
    // second half is in registers.
    const int sub = warp & 3;
    const uint32_t tD = tmem + (static_cast<uint32_t>(32 * sub) << 16);
    const uint32_t stage = sO + sub * C::O_WARP_BYTES;
    int n = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++n) {
      const int tw = tile % a.tiles_w, tt = tile / a.tiles_w;
      // the 128 features of a weight tile lie in one of q, k, v (widths are
      // multiples of 128)
      int col = tw * C::BW + 32 * sub;
      const CUtensorMap* map = &tmQ;
      if (col >= a.width0) {
        col -= a.width0;
        map = &tmK;
        if (col >= a.width1) {
          col -= a.width1;
          map = &tmV;
        }
      }
      if (!warp_wait(smem_u32(&bar_acc_full), n & 1, wc, 65)) break;
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t pk[64];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t r[16];
          tmem_ld16(tD + 128 * h + 16 * c, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 8; ++i)
            pk[8 * c + i] = pack_bf16x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
        }
        if (h == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&bar_acc_empty));
        }
        // the previous store from the staging area has finished reading it
        if (lane == 0) bulk_wait_read_all();
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 128; ++j)
          st_shared_u16(stage + j * 64 + lane * 2, static_cast<uint16_t>(pk[j >> 1] >> (16 * (j & 1))));
        fence_proxy_async_smem();
        __syncwarp();
        const int t0 = tt * C::BT + 128 * h;
        if (lane == 0 && t0 < a.M) {
          tma_store_2d(map, stage, col, t0);
          bulk_commit_group();
        }
        __syncwarp();
      }
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Dequantization alone: W' bf16 [rows, K] (the operand a separate GEMM would
// read).  One thread per 8 elements (one 32-bit word of codes); a warp covers
// 256 consecutive elements, so loads (128 B) and stores (512 B) coalesce.
__global__ void __launch_bounds__(256) s2_nf4_dequant_kernel(const uint32_t* codes, const int8_t* sq,
                                                             const float* c2, __nv_bfloat16* w, long long n_words,
                                                             Nf4Levels lv) {
  const int lane = threadIdx.x & 31;
  const float table = lane_level(lv, lane);
  const long long warps = static_cast<long long>(gridDim.x) * 8;
  for (long long base = (blockIdx.x * 8LL + (threadIdx.x >> 5)) * 32; base < n_words; base += warps * 32) {
    // warp-uniform loop: every lane takes part in the shuffles
    const long long e = base + lane;
    const bool valid = e < n_words;
    const uint32_t wd = valid ? __ldg(codes + e) : 0u;
    const long long blk = valid ? (e >> 3) : 0;  // 64-element block
    const float sc = valid ? static_cast<float>(sq[blk]) * __ldg(c2 + (blk >> 8)) / 127.f : 0.f;
    const uint64_t sc2 = f2_pack(sc, sc);
    uint32_t pk[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const float lo = warp_lut16(table, wd >> (8 * p));
      const float hi = warp_lut16(table, wd >> (8 * p + 4));
      pk[p] = f2_to_bf16x2(f2_mul(f2_pack(lo, hi), sc2));
    }
    if (valid) *reinterpret_cast<uint4*>(w + e * 8) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
}

template <int NS, int DQW>
cudaError_t launch_nf4_qkv_variant(const CUtensorMap& tx, const CUtensorMap& tc, const CUtensorMap* to,
                                   const Nf4Args& a, int num_sms, cudaStream_t stream) {
  using C = Nf4Cfg<NS, DQW>;
  cudaError_t ea = cudaFuncSetAttribute(s2_nf4_qkv_kernel<NS, DQW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        C::SMEM_BYTES);
  if (ea != cudaSuccess) return ea;
  const int ntiles = a.tiles_w * a.tiles_t;
  const int grid = ntiles < num_sms ? ntiles : num_sms;
  prof_before(stream, kKernelNf4Qkv);
  s2_nf4_qkv_kernel<NS, DQW><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tx, tc, to[0], to[1], to[2], a);
  cudaError_t e = cudaGetLastError();
  prof_after(stream);
  return e;
}

// stages: pipeline depth 4 or 5; dq_warps: dequantization warps, 8 or 12
cudaError_t launch_nf4_qkv(const CUtensorMap& tx, const CUtensorMap& tc, const CUtensorMap* to, const Nf4Args& a,
                           int num_sms, cudaStream_t stream, int stages, int dq_warps) {
  if (stages == 5 && dq_warps == 8) return launch_nf4_qkv_variant<5, 8>(tx, tc, to, a, num_sms, stream);
  if (stages == 5 && dq_warps == 12) return launch_nf4_qkv_variant<5, 12>(tx, tc, to, a, num_sms, stream);
  if (stages == 4 && dq_warps == 8) return launch_nf4_qkv_variant<4, 8>(tx, tc, to, a, num_sms, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_nf4_dequant(const void* codes, const int8_t* sq, const float* c2, void* w, long long n_words,
                               const Nf4Levels& lv, int num_sms, cudaStream_t stream) {
  const long long warps_needed = (n_words + 31) / 32;
  const long long blocks = (warps_needed + 7) / 8;
  const int grid = static_cast<int>(blocks < 8LL * num_sms ? blocks : 8LL * num_sms);
  prof_before(stream, kKernelNf4Dequant);
  s2_nf4_dequant_kernel<<<grid, 256, 0, stream>>>(static_cast<const uint32_t*>(codes), sq, c2,
                                                  static_cast<__nv_bfloat16*>(w), n_words, lv);
  cudaError_t e = cudaGetLastError();
  prof_after(stream);
  return e;
}

}  // namespace s2
