// S2-Attn forward for sm_100a: tcgen05 UMMA with TMEM accumulators, TMA-fed
// K/V ring, online softmax in fp32 with one query row per thread.
//
// One CTA computes one 128-row query tile of one (batch, head).  Its key/value
// tiles run from the start of the tile's rolled group up to the diagonal tile;
// tiles above the diagonal and outside the group are never touched (LongQLoRA
// community post, section 03: attention only inside each group; section 04:
// causal next-token objective).
//
// Warp roles (320 threads):
//   warp 0      TMA producer: Q once, then K_j / V_j into a STAGES-deep ring.
//   warp 1      TMEM owner and UMMA issuer: S_j = Q K_j^T (double-buffered in
//               TMEM), O += P_j V_j with P_j read from TMEM.
//   warps 2..9  softmax: two threads per query row (warps 2..5 the first 64
//               key columns of a tile, warps 6..9 the last 64); S from TMEM,
//               running max and sum, P (bf16) written back over S, O rescaled
//               in TMEM only when the running max grows by more than 2^8,
//               epilogue.
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
  // K and V tiles share one ring of slots, filled in the order K0 V0 K1 V1 ...;
  // a K slot is released as soon as its S UMMA completes.
  static constexpr int SLOTS = (D == 64) ? 8 : 5;
  static constexpr int ATOM_BYTES = kTile * 128;  // one 64-column slab of a 128-row tile
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int OFF_KV = Q_BYTES;
  static constexpr int SMEM_BYTES = OFF_KV + SLOTS * KV_BYTES + 1024;  // + alignment slack
  static constexpr uint32_t TM_O = 256;
  static constexpr int THREADS = 320;
};

// Cubic for 2^f on [-1/2, 1/2], minimax in relative error (derived by
// derive_exp2_poly.py in this directory; max relative error 7.5e-5 in float32).
constexpr float kExp2C0 = 9.999280572e-01f;
constexpr float kExp2C1 = 6.932609677e-01f;
constexpr float kExp2C2 = 2.426111251e-01f;
constexpr float kExp2C3 = 5.517166853e-02f;

// 2^x on the FMA pipe (Cody-Waite split x = n + f, n = round(x), f in
// [-1/2, 1/2]; 2^n added to the exponent field).  x is clamped below at -126
// so the result stays a (tiny) non-negative float; inputs here are <= 8.
__device__ __forceinline__ float exp2_fma(float x) {
  x = fmaxf(x, -126.f);
  const float t = x + 12582912.f;  // 1.5 * 2^23: round(x) lands in the low mantissa bits
  const float f = x - (t - 12582912.f);
  const float p = fmaf(fmaf(fmaf(kExp2C3, f, kExp2C2), f, kExp2C1), f, kExp2C0);
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// The same on a packed pair, with f32x2 arithmetic.
__device__ __forceinline__ uint64_t exp2_fma2(uint64_t x) {
  const uint64_t xc = f2_pack(fmaxf(f2_lo(x), -126.f), fmaxf(f2_hi(x), -126.f));
  const uint64_t t = f2_add(xc, f2_pack(12582912.f, 12582912.f));
  const uint64_t f = f2_add(xc, f2_add(t, f2_pack(-12582912.f, -12582912.f)) ^ 0x8000000080000000ull);
  uint64_t p = f2_fma(f2_pack(kExp2C3, kExp2C3), f, f2_pack(kExp2C2, kExp2C2));
  p = f2_fma(p, f, f2_pack(kExp2C1, kExp2C1));
  p = f2_fma(p, f, f2_pack(kExp2C0, kExp2C0));
  const uint32_t lo = __float_as_uint(f2_lo(p)) + (static_cast<uint32_t>(t) << 23);
  const uint32_t hi = __float_as_uint(f2_hi(p)) + (static_cast<uint32_t>(t >> 32) << 23);
  return (static_cast<uint64_t>(hi) << 32) | lo;
}

// P for 64 scores of one query row: p = 2^(s * sl2 - m), packed to bf16
// pairs in pk; returns the fp32 sum.  Arguments and sums use packed f32x2
// arithmetic; one pair in four takes its exponentials on the FMA pipe
// (exp2_fma2), the rest on the MUFU (ex2.approx), which balances the pipes.
__device__ __forceinline__ float softmax_row64(const uint32_t (&sr)[2][32], float sl2, float m,
                                               uint32_t (&pk)[32]) {
  const uint64_t sc2 = f2_pack(sl2, sl2), nm2 = f2_pack(-m, -m);
  uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    const uint64_t x = f2_fma(f2_pack(__uint_as_float(sr[(2 * c) >> 5][(2 * c) & 31]),
                                      __uint_as_float(sr[(2 * c + 1) >> 5][(2 * c + 1) & 31])),
                              sc2, nm2);
    uint64_t p;
    if ((c & 3) == 0) {
      p = exp2_fma2(x);
    } else {
      p = f2_pack(ex2_approx(f2_lo(x)), ex2_approx(f2_hi(x)));
    }
    pk[c] = f2_to_bf16x2(p);
    acc[c & 3] = f2_add(acc[c & 3], p);
  }
  const uint64_t s = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
  return f2_lo(s) + f2_hi(s);
}

template <int D>
__global__ void __launch_bounds__(320, 1)
    s2_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const FwdArgs a) {
  using C = FwdCfg<D>;
  constexpr int NS = C::SLOTS;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) uint64_t bar_q, bar_full[NS], bar_empty[NS], bar_s[2], bar_p[2], bar_x[2],
      bar_l, bar_o, bar_drain;
  __shared__ float red_max[2][2][kTile];  // [tile parity][half][row] partial row maxima
  __shared__ float red_sum[2][kTile];     // [half][row] partial row sums
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
  auto slot_addr = [&](int s) { return sQ + C::OFF_KV + s * C::KV_BYTES; };

  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar_q), 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(smem_u32(&bar_full[s]), 1);
      mbar_init(smem_u32(&bar_empty[s]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bar_s[i]), 1);
      mbar_init(smem_u32(&bar_p[i]), 8);  // one elected arrival per softmax warp
      mbar_init(smem_u32(&bar_x[i]), 8);
    }
    mbar_init(smem_u32(&bar_l), 8);
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
    // (whole warp converged; one elected lane issues the copies)
    if (elect_one()) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(smem_u32(&bar_q), C::Q_BYTES);
      for (int c = 0; c < D / 64; ++c)
        tma_load_4d(sQ + c * C::ATOM_BYTES, &tmQ, smem_u32(&bar_q), c * 64, w.h, tq0, w.b);
    }
    __syncwarp();
    int issued = 0;
    for (int L = 0; L < 2 * nkv; ++L) {  // load L: K_{L/2} (even) or V_{L/2} (odd)
      const int s = L % NS, n = L / NS;
      if (n > 0 && !warp_wait(smem_u32(&bar_empty[s]), (n - 1) & 1, wc, 10)) break;
      const int tk0 = original_row(d, w.g * d.G + (L >> 1) * kTile, sh);
      const CUtensorMap* map = (L & 1) ? &tmV : &tmK;
      if (elect_one()) {
        mbar_arrive_expect_tx(smem_u32(&bar_full[s]), C::KV_BYTES);
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(slot_addr(s) + c * C::ATOM_BYTES, map, smem_u32(&bar_full[s]), c * 64, w.kvh,
                      tk0, w.b);
      }
      __syncwarp();
      ++issued;
    }
    if (*wc.abort && lane == 0) {
      // never leave copies in flight into shared memory: wait (bounded) for
      // the last fill of every slot and for Q
      drain_wait(smem_u32(&bar_q), 0);
      for (int s = 0; s < NS && s < issued; ++s)
        drain_wait(smem_u32(&bar_full[s]), ((issued - 1 - s) / NS) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer
    // (whole warp converged; one elected lane issues each batch)
    const uint32_t idS = make_idesc_bf16(128, C::BN, 0, 0);  // Q K-major, K K-major
    const uint32_t idO = make_idesc_bf16(128, D, 0, 1);      // P from TMEM, V MN-major
    // operand descriptors: built once, then advanced by constants
    const uint64_t dQ0 = make_sdesc_sw128(sQ, 16, 1024);                      // K-major
    const uint64_t dK0 = make_sdesc_sw128(slot_addr(0), 16, 1024);            // K-major
    const uint64_t dV0 = make_sdesc_sw128(slot_addr(0), C::ATOM_BYTES, 1024);  // MN-major
    // S_j = Q K_j^T into S buffer j&1; releases K_j's slot when done
    auto issue_qk = [&](int j) -> bool {
      const int L = 2 * j, s = L % NS;
      if (!warp_wait(smem_u32(&bar_full[s]), (L / NS) & 1, wc, 22)) return false;
      tc_fence_after();
      const uint64_t dk = sdesc_advance(dK0, s * C::KV_BYTES);
      const uint32_t tS = tmem + (j & 1) * 128;
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::ATOM_BYTES + (kk & 3) * 32;
          umma_ss(tS, sdesc_advance(dQ0, off), sdesc_advance(dk, off), idS, kk > 0);
        }
        umma_commit(smem_u32(&bar_s[j & 1]));
        umma_commit(smem_u32(&bar_empty[s]));
      }
      __syncwarp();
      return true;
    };
    bool ok = warp_wait(smem_u32(&bar_q), 0, wc, 20) && issue_qk(0);
    for (int j = 0; ok && j < nkv; ++j) {
      if (j + 1 < nkv && !issue_qk(j + 1)) break;
      const int L = 2 * j + 1, s = L % NS;
      if (!warp_wait(smem_u32(&bar_p[j & 1]), (j >> 1) & 1, wc, 23)) break;
      if (!warp_wait(smem_u32(&bar_full[s]), (L / NS) & 1, wc, 24)) break;
      tc_fence_after();
      const uint32_t tP = tmem + (j & 1) * 128;
      const uint64_t dv = sdesc_advance(dV0, s * C::KV_BYTES);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk)
          umma_ts(tmem + C::TM_O, tP + kk * 8, sdesc_advance(dv, kk * 2048), idO, (j > 0 || kk > 0));
        umma_commit(smem_u32(&bar_o));
        umma_commit(smem_u32(&bar_empty[s]));
      }
      __syncwarp();
    }
    // every issued UMMA completes before TMEM is released
    if (elect_one()) {
      umma_commit(smem_u32(&bar_drain));
      drain_wait(smem_u32(&bar_drain), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    // Two warpgroups share every query row: warps 2..5 take key columns
    // [0,64) of each tile, warps 6..9 columns [64,128).  The two halves of a
    // row exchange their partial maxima through shared memory each tile (and
    // their partial sums once at the end); both then take identical decisions.
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int half = (warp - 2) >> 2;
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
      uint32_t sr[2][32];
      tmem_ld32(tS + half * 64, sr[0]);
      tmem_ld32(tS + half * 64 + 32, sr[1]);
      tmem_wait_ld();
      if (j == nkv - 1) {  // diagonal tile: keys after the query are masked
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (half * 64 + c > row) sr[c >> 5][c & 31] = __float_as_uint(neg_inf());
      }
      float m4[4] = {neg_inf(), neg_inf(), neg_inf(), neg_inf()};
#pragma unroll
      for (int c = 0; c < 64; ++c) m4[c & 3] = fmaxf(m4[c & 3], __uint_as_float(sr[c >> 5][c & 31]));
      const float mh = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      // exchange partial maxima with the other half of the row (double-buffered
      // slot).  From the second tile on the exchange completes in the
      // background: P is computed against the running max first and redone
      // only if the row max grew by more than 2^8 (rare after the first tiles).
      red_max[j & 1][half][row] = mh;
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar_x[j & 1]));
      auto exchange = [&]() -> bool {
        bool ok2 = true;
        if (lane == 0) ok2 = mbar_wait(smem_u32(&bar_x[j & 1]), (j >> 1) & 1, wc, 33);
        return __shfl_sync(0xffffffffu, ok2, 0);
      };
      if (j == 0) {
        if (!exchange()) { ok = false; break; }
        m_run = fmaxf(mh, red_max[0][half ^ 1][row]) * sl2;
      }
      uint32_t pk[32];
      float rs = softmax_row64(sr, sl2, m_run, pk);
      float alpha = 1.f;
      bool resc = false;
      if (j > 0) {
        if (!exchange()) { ok = false; break; }
        const float mx = fmaxf(mh, red_max[j & 1][half ^ 1][row]) * sl2;
        if (mx > m_run + 8.f) {
          alpha = ex2_approx(m_run - mx);
          m_run = mx;
          resc = true;
          rs = softmax_row64(sr, sl2, m_run, pk);
        }
      }
      l_run = l_run * alpha + rs;
      // P (bf16) over the first 64 columns of this S buffer; both halves read
      // their S columns before the exchange above, so no write races a read
      tmem_st32(tS + half * 32, pk);
      if (__any_sync(0xffffffffu, resc)) {
        // O holds P_{j-1} V_{j-1} only once that UMMA has completed
        if (lane == 0) ok = mbar_wait(smem_u32(&bar_o), (j - 1) & 1, wc, 31);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          uint32_t o[32];
          const uint32_t to = tmem + lane_off + C::TM_O + half * (D / 2) + c * 32;
          tmem_ld32(to, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(to, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar_p[j & 1]));
    }
    // ------------------------------------------------------------ epilogue
    if (ok) {
      red_sum[half][row] = l_run;
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(&bar_l));
        ok = mbar_wait(smem_u32(&bar_l), 0, wc, 34) && mbar_wait(smem_u32(&bar_o), (nkv - 1) & 1, wc, 32);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
    }
    if (ok) {
      tc_fence_after();
      const float l_tot = l_run + red_sum[half ^ 1][row];
      const float inv_l = 1.f / l_tot;
      const int t = tq0 + row;
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.o) +
                            ((static_cast<size_t>(w.b) * d.N + t) * d.H + w.h) * D + half * (D / 2);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_off + C::TM_O + half * (D / 2) + c * 32, o);
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
      if (half == 0)
        a.lse[(static_cast<size_t>(w.b) * d.H + w.h) * d.N + t] =
            (m_run + __log2f(l_tot)) * 0.69314718055994530942f;
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

// Test hook: the FMA-pipe exp2 next to CUDA's exp2f on the same inputs.
// (pairs go through the packed form the softmax uses; an odd last element
// through the scalar form)
__global__ void s2_exp2_selftest_kernel(const float* x, float* y_poly, float* y_ref, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    const uint64_t p = exp2_fma2(f2_pack(x[i], x[i + 1]));
    y_poly[i] = f2_lo(p);
    y_poly[i + 1] = f2_hi(p);
    y_ref[i] = exp2f(x[i]);
    y_ref[i + 1] = exp2f(x[i + 1]);
  } else if (i < n) {
    y_poly[i] = exp2_fma(x[i]);
    y_ref[i] = exp2f(x[i]);
  }
}

cudaError_t launch_exp2_selftest(const float* x, float* y_poly, float* y_ref, int n, cudaStream_t stream) {
  s2_exp2_selftest_kernel<<<((n + 1) / 2 + 255) / 256, 256, 0, stream>>>(x, y_poly, y_ref, n);
  return cudaGetLastError();
}

template cudaError_t launch_fwd<64>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                    const FwdArgs&, cudaStream_t);
template cudaError_t launch_fwd<128>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                     const FwdArgs&, cudaStream_t);

}  // namespace s2
