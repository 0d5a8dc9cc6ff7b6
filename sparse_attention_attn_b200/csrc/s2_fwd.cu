// S2-Attn forward for sm_100a: tcgen05 UMMA with TMEM accumulators, TMA-fed
// K/V ring, online softmax in fp32 with one query row per thread.
//
// One CTA computes one 128-row query tile of one (batch, head).  Its key/value
// tiles run from the start of the tile's rolled group up to the diagonal tile;
// tiles above the diagonal and outside the group are never touched (LongQLoRA
// community post, section 03: attention only inside each group; section 04:
// causal next-token objective).
//
// Warp roles (192 threads):
//   warp 0      TMA producer: Q once, then K_j / V_j into a STAGES-deep ring.
//   warp 1      TMEM owner and UMMA issuer: S_j = Q K_j^T (double-buffered in
//               TMEM), O += P_j V_j with P_j read from TMEM.
//   warps 2..5  softmax: thread = query row; S row from TMEM, running max and
//               sum, P (bf16) written back over S, O rescaled in TMEM only
//               when the running max grows by more than 2^8, epilogue.
//
// TMEM (512 columns): S buffers at [0,128) and [128,256) (P over their first
// 64 columns), O at [256, 256 + D).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "s2_common.cuh"
#include "s2_ptx.cuh"

namespace s2 {

template <int D>
struct FwdCfg {
  static constexpr int BM = kTile, BN = kTile;
  static constexpr int STAGES = (D == 64) ? 4 : 3;
  static constexpr int ATOM_BYTES = kTile * 128;  // one 64-column slab of a 128-row tile
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int OFF_K = Q_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * KV_BYTES;
  static constexpr int SMEM_BYTES = OFF_V + STAGES * KV_BYTES + 1024;  // + alignment slack
  static constexpr uint32_t TM_O = 256;
  static constexpr int THREADS = 192;
};

template <int D>
__global__ void __launch_bounds__(192, 1)
    s2_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const FwdArgs a) {
  using C = FwdCfg<D>;
  constexpr int ST = C::STAGES;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) uint64_t bar_q, bar_k[ST], bar_v[ST], bar_empty[ST], bar_s[2], bar_p[2],
      bar_o, bar_drain;
  __shared__ uint32_t tmem_slot;
  __shared__ uint32_t abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Dims& d = a.d;
  const TileWork w = decode_q_tile(d, blockIdx.x);
  const int sh = shift_of_head(d, w.h);
  const int r0 = w.g * d.G + w.tile * kTile;  // rolled first row of this query tile
  const int tq0 = original_row(d, r0, sh);     // its original row (the tile never wraps)
  const int nkv = w.tile + 1;
  WaitCtx wc{&abort_flag, a.status, a.wait_limit_ns};

  const uint32_t sQ = smem_u32(smem);
  auto sK = [&](int s) { return sQ + C::OFF_K + s * C::KV_BYTES; };
  auto sV = [&](int s) { return sQ + C::OFF_V + s * C::KV_BYTES; };

  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar_q), 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(smem_u32(&bar_k[s]), 1);
      mbar_init(smem_u32(&bar_v[s]), 1);
      mbar_init(smem_u32(&bar_empty[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bar_s[i]), 1);
      mbar_init(smem_u32(&bar_p[i]), 128);
    }
    mbar_init(smem_u32(&bar_o), 1);
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
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(smem_u32(&bar_q), C::Q_BYTES);
      for (int c = 0; c < D / 64; ++c)
        tma_load_4d(sQ + c * C::ATOM_BYTES, &tmQ, smem_u32(&bar_q), c * 64, w.h, tq0, w.b);
      int issued = 0;
      for (int j = 0; j < nkv; ++j) {
        const int s = j % ST, n = j / ST;
        if (n > 0 && !mbar_wait(smem_u32(&bar_empty[s]), (n - 1) & 1, wc, 10)) break;
        const int tk0 = original_row(d, w.g * d.G + j * kTile, sh);
        mbar_arrive_expect_tx(smem_u32(&bar_k[s]), C::KV_BYTES);
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(sK(s) + c * C::ATOM_BYTES, &tmK, smem_u32(&bar_k[s]), c * 64, w.kvh, tk0,
                      w.b);
        mbar_arrive_expect_tx(smem_u32(&bar_v[s]), C::KV_BYTES);
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(sV(s) + c * C::ATOM_BYTES, &tmV, smem_u32(&bar_v[s]), c * 64, w.kvh, tk0,
                      w.b);
        ++issued;
      }
      if (*wc.abort) {
        // never leave copies in flight into shared memory: wait (bounded) for
        // the last fill of every stage and for Q
        drain_wait(smem_u32(&bar_q), 0);
        for (int s = 0; s < ST && s < issued; ++s) {
          const int last = (issued - 1 - s) / ST;
          drain_wait(smem_u32(&bar_k[s]), last & 1);
          drain_wait(smem_u32(&bar_v[s]), last & 1);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      const uint32_t idS = make_idesc_bf16(128, C::BN, 0, 0);  // Q K-major, K K-major
      const uint32_t idO = make_idesc_bf16(128, D, 0, 1);      // P from TMEM, V MN-major
      auto issue_qk = [&](uint32_t tS, uint32_t k_base) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::ATOM_BYTES + (kk & 3) * 32;
          umma_ss(tS, make_sdesc_sw128(sQ + off, 16, 1024), make_sdesc_sw128(k_base + off, 16, 1024),
                  idS, kk > 0);
        }
      };
      bool ok = mbar_wait(smem_u32(&bar_q), 0, wc, 20) && mbar_wait(smem_u32(&bar_k[0]), 0, wc, 21);
      if (ok) {
        tc_fence_after();
        issue_qk(tmem, sK(0));
        umma_commit(smem_u32(&bar_s[0]));
      }
      for (int j = 0; ok && j < nkv; ++j) {
        const int s = j % ST;
        if (j + 1 < nkv) {
          const int s1 = (j + 1) % ST;
          if (!mbar_wait(smem_u32(&bar_k[s1]), ((j + 1) / ST) & 1, wc, 22)) break;
          tc_fence_after();
          issue_qk(tmem + ((j + 1) & 1) * 128, sK(s1));
          umma_commit(smem_u32(&bar_s[(j + 1) & 1]));
        }
        if (!mbar_wait(smem_u32(&bar_p[j & 1]), (j >> 1) & 1, wc, 23)) break;
        if (!mbar_wait(smem_u32(&bar_v[s]), (j / ST) & 1, wc, 24)) break;
        tc_fence_after();
        const uint32_t tP = tmem + (j & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk)
          umma_ts(tmem + C::TM_O, tP + kk * 8,
                  make_sdesc_sw128(sV(s) + kk * 2048, C::ATOM_BYTES, 1024), idO, (j > 0 || kk > 0));
        umma_commit(smem_u32(&bar_o));
        umma_commit(smem_u32(&bar_empty[s]));
      }
      // every issued UMMA completes before TMEM is released
      umma_commit(smem_u32(&bar_drain));
      drain_wait(smem_u32(&bar_drain), 0);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float sl2 = a.scale_log2;
    float m_run = 0.f, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      const uint32_t tS = tmem + lane_off + (j & 1) * 128;
      if (lane == 0) ok = mbar_wait(smem_u32(&bar_s[j & 1]), (j >> 1) & 1, wc, 30);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, sr[c]);
      tmem_wait_ld();
      const bool diag = (j == nkv - 1);
      float mx = neg_inf();
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        float v = __uint_as_float(sr[c >> 5][c & 31]);
        if (diag && c > row) v = neg_inf();
        sr[c >> 5][c & 31] = __float_as_uint(v);
        mx = fmaxf(mx, v);
      }
      mx *= sl2;
      float alpha = 1.f;
      bool resc = false;
      if (j == 0) {
        m_run = mx;
      } else if (mx > m_run + 8.f) {
        alpha = ex2_approx(m_run - mx);
        m_run = mx;
        resc = true;
      }
      uint32_t pk[2][32];
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float p0 = ex2_approx(fmaf(__uint_as_float(sr[(2 * c) >> 5][(2 * c) & 31]), sl2, -m_run));
        const float p1 =
            ex2_approx(fmaf(__uint_as_float(sr[(2 * c + 1) >> 5][(2 * c + 1) & 31]), sl2, -m_run));
        pk[c >> 5][c & 31] = pack_bf16x2(p0, p1);
        rs += p0 + p1;
      }
      l_run = l_run * alpha + rs;
      tmem_st32(tS, pk[0]);
      tmem_st32(tS + 32, pk[1]);
      if (__any_sync(0xffffffffu, resc)) {
        // O holds P_{j-1} V_{j-1} only once that UMMA has completed
        if (lane == 0) ok = mbar_wait(smem_u32(&bar_o), (j - 1) & 1, wc, 31);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_off + C::TM_O + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tmem + lane_off + C::TM_O + c * 32, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&bar_p[j & 1]));
    }
    // ------------------------------------------------------------ epilogue
    if (ok) {
      if (lane == 0) ok = mbar_wait(smem_u32(&bar_o), (nkv - 1) & 1, wc, 32);
      ok = __shfl_sync(0xffffffffu, ok, 0);
    }
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / l_run;
      const int t = tq0 + row;
      __nv_bfloat16* orow =
          static_cast<__nv_bfloat16*>(a.o) + ((static_cast<size_t>(w.b) * d.N + t) * d.H + w.h) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_off + C::TM_O + c * 32, o);
        tmem_wait_ld();
        uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(o[8 * q + 0]) * inv_l, __uint_as_float(o[8 * q + 1]) * inv_l);
          v.y = pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv_l, __uint_as_float(o[8 * q + 3]) * inv_l);
          v.z = pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv_l, __uint_as_float(o[8 * q + 5]) * inv_l);
          v.w = pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv_l, __uint_as_float(o[8 * q + 7]) * inv_l);
          dst[q] = v;
        }
      }
      a.lse[(static_cast<size_t>(w.b) * d.H + w.h) * d.N + t] =
          (m_run + __log2f(l_run)) * 0.69314718055994530942f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D>
cudaError_t launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const FwdArgs& a, cudaStream_t stream) {
  using C = FwdCfg<D>;
  cudaError_t ea = cudaFuncSetAttribute(s2_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        C::SMEM_BYTES);
  if (ea != cudaSuccess) return ea;
  const int grid = a.d.B * a.d.H * a.d.n_groups * a.d.tiles;
  prof_before(stream, kKernelFwd);
  s2_fwd_kernel<D><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, a);
  cudaError_t e = cudaGetLastError();
  prof_after(stream);
  return e;
}

template cudaError_t launch_fwd<64>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                    const FwdArgs&, cudaStream_t);
template cudaError_t launch_fwd<128>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                     const FwdArgs&, cudaStream_t);

}  // namespace s2
