// Rotary position embedding with Position Interpolation (LongQLoRA community
// post: LLaMA uses rotary position encoding, section 02; Position
// Interpolation shrinks its rotation angles to reach 8192 tokens, section 04),
// applied to q and k at their original positions before S2 attention.
//
// Pair i of a head (elements i and i + D/2) at token t turns by
//   a(t, i) = t * s * base^(-2i/D),   s = L_train / L_target.
// At 100K tokens a reaches ~1e5 radians, beyond what fp32 sin/cos (or an fp32
// product t * s * f) can resolve, so the table kernel forms the angle and its
// cosine and sine in fp64 and stores fp32 (cos, sin) pairs, [N][D/2][2]; the
// rotation kernels and the fused backward epilogues read that table.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "s2_common.cuh"
#include "s2_ptx.cuh"

namespace s2 {

__global__ void __launch_bounds__(256) s2_rope_table_kernel(float2* table, int N, int half, double pos_scale,
                                                            double log_base) {
  const long long n = static_cast<long long>(N) * half;
  for (long long e = blockIdx.x * 256LL + threadIdx.x; e < n; e += static_cast<long long>(gridDim.x) * 256) {
    const int t = static_cast<int>(e / half), i = static_cast<int>(e - static_cast<long long>(t) * half);
    const double freq = exp(-static_cast<double>(i) / half * log_base);  // base^(-2i/D)
    const double a = static_cast<double>(t) * pos_scale * freq;
    double s, c;
    sincos(a, &s, &c);
    table[e] = make_float2(static_cast<float>(c), static_cast<float>(s));
  }
}

// One thread per (batch, token, 8 pairs, group of up to 4 heads): the 8
// (cos, sin) pairs of its token stay in registers while it rotates its heads;
// per head it reads 8 values of each half of the row and writes the rotated
// 16.  `inverse` turns by -a.  x and out may be the same buffer.
template <int D>
__global__ void __launch_bounds__(256) s2_rope_apply_kernel(const __nv_bfloat16* x, __nv_bfloat16* out,
                                                            const float2* table, int B, int N, int heads,
                                                            int inverse) {
  constexpr int CH = D / 16;  // 8-pair chunks per head
  constexpr int HG = 4;       // heads per thread
  const int ngrp = (heads + HG - 1) / HG;
  const long long n = static_cast<long long>(B) * N * ngrp * CH;
  const float sg = inverse ? -1.f : 1.f;
  for (long long e = blockIdx.x * 256LL + threadIdx.x; e < n; e += static_cast<long long>(gridDim.x) * 256) {
    // consecutive threads: chunks of one head group, then the groups of a token
    const int ch = static_cast<int>(e % CH);
    const long long r = e / CH;
    const int hg = static_cast<int>(r % ngrp);
    const long long bt = r / ngrp;  // b * N + t
    const int t = static_cast<int>(bt % N);
    const float4* tp = reinterpret_cast<const float4*>(table + static_cast<size_t>(t) * (D / 2) + ch * 8);
    float c[8], s[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 v = tp[j];
      c[2 * j] = v.x;
      s[2 * j] = v.y * sg;
      c[2 * j + 1] = v.z;
      s[2 * j + 1] = v.w * sg;
    }
    const size_t row = static_cast<size_t>(bt) * heads * D;
    const int h0 = hg * HG, h1 = h0 + HG < heads ? h0 + HG : heads;
    uint4 u1[HG], u2[HG];
#pragma unroll
    for (int k = 0; k < HG; ++k) {
      if (h0 + k < h1) {
        const size_t o1 = row + static_cast<size_t>(h0 + k) * D + ch * 8;
        u1[k] = *reinterpret_cast<const uint4*>(x + o1);
        u2[k] = *reinterpret_cast<const uint4*>(x + o1 + D / 2);
      }
    }
#pragma unroll
    for (int k = 0; k < HG; ++k) {
      if (h0 + k >= h1) continue;
      const size_t o1 = row + static_cast<size_t>(h0 + k) * D + ch * 8;
      const uint32_t a1[4] = {u1[k].x, u1[k].y, u1[k].z, u1[k].w}, a2[4] = {u2[k].x, u2[k].y, u2[k].z, u2[k].w};
      uint32_t r1[4], r2[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 x1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&a1[j]));
        const float2 x2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&a2[j]));
        const int k0 = 2 * j, k1 = 2 * j + 1;
        r1[j] = pack_bf16x2(fmaf(x1.x, c[k0], -x2.x * s[k0]), fmaf(x1.y, c[k1], -x2.y * s[k1]));
        r2[j] = pack_bf16x2(fmaf(x1.x, s[k0], x2.x * c[k0]), fmaf(x1.y, s[k1], x2.y * c[k1]));
      }
      *reinterpret_cast<uint4*>(out + o1) = make_uint4(r1[0], r1[1], r1[2], r1[3]);
      *reinterpret_cast<uint4*>(out + o1 + D / 2) = make_uint4(r2[0], r2[1], r2[2], r2[3]);
    }
  }
}

cudaError_t launch_rope_table(float* table, int N, int D, double pos_scale, double base, int num_sms,
                              cudaStream_t stream) {
  const long long n = static_cast<long long>(N) * (D / 2);
  const long long blocks = (n + 255) / 256;
  const int grid = static_cast<int>(blocks < 8LL * num_sms ? blocks : 8LL * num_sms);
  s2_rope_table_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<float2*>(table), N, D / 2, pos_scale,
                                                 log(base));
  return cudaGetLastError();
}

cudaError_t launch_rope_apply(const void* x, void* out, const float* table, int B, int N, int heads, int D,
                              int inverse, int num_sms, cudaStream_t stream) {
  const long long n = static_cast<long long>(B) * N * ((heads + 3) / 4) * (D / 16);
  const long long blocks = (n + 255) / 256;
  const int grid = static_cast<int>(blocks < 16LL * num_sms ? blocks : 16LL * num_sms);
  const auto* xin = static_cast<const __nv_bfloat16*>(x);
  auto* xo = static_cast<__nv_bfloat16*>(out);
  const auto* tb = reinterpret_cast<const float2*>(table);
  prof_before(stream, kKernelRope);
  if (D == 64)
    s2_rope_apply_kernel<64><<<grid, 256, 0, stream>>>(xin, xo, tb, B, N, heads, inverse);
  else
    s2_rope_apply_kernel<128><<<grid, 256, 0, stream>>>(xin, xo, tb, B, N, heads, inverse);
  cudaError_t e = cudaGetLastError();
  prof_after(stream);
  return e;
}

}  // namespace s2
