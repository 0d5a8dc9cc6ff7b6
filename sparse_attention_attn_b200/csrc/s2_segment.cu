// Log-sum-exp merge of two attention pieces over disjoint key sets (the
// detached earlier segment and the chunk's own keys of chunk-wise training:
// HGA digest, segment-wise backpropagation with detached older KV; SeCO /
// SpaCO digest, chunk-wise optimisation):
//   lse = log(exp(lse_a) + exp(lse_b)),
//   o   = exp(lse_a - lse) o_a + exp(lse_b - lse) o_b.
// One thread per 8 values of a (batch, row, head); the D/8 threads of a row
// are lanes of one warp, and since N is a multiple of 128 every warp's lanes
// run the same number of loop iterations (the __syncwarp below is safe).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "s2_common.cuh"
#include "s2_ptx.cuh"

namespace s2 {

template <int D>
__global__ void __launch_bounds__(256) s2_lse_merge_kernel(const __nv_bfloat16* oa, const float* la,
                                                           const __nv_bfloat16* ob, const float* lb,
                                                           __nv_bfloat16* o, float* lse, int B, int H, int N) {
  constexpr int CH = D / 8;  // threads per row
  const long long n = static_cast<long long>(B) * N * H * CH;
  for (long long e = blockIdx.x * 256LL + threadIdx.x; e < n; e += static_cast<long long>(gridDim.x) * 256) {
    const long long row = e / CH;  // (b * N + t) * H + h
    const int c = static_cast<int>(e - row * CH);
    const int h = static_cast<int>(row % H);
    const long long bt = row / H;
    const int t = static_cast<int>(bt % N), b = static_cast<int>(bt / N);
    const size_t li = (static_cast<size_t>(b) * H + h) * N + t;
    const float xa = la[li], xb = lb[li];
    const float m = fmaxf(xa, xb);
    // a piece with lse = -inf (no visible key) has weight 0
    const float ea = xa == m ? 1.f : __expf(xa - m), eb = xb == m ? 1.f : __expf(xb - m);
    const float inv = 1.f / (ea + eb);
    const float wa = ea * inv, wb = eb * inv;
    const size_t oi = static_cast<size_t>(row) * D + c * 8;
    const uint4 ua = *reinterpret_cast<const uint4*>(oa + oi);
    const uint4 ub = *reinterpret_cast<const uint4*>(ob + oi);
    const uint32_t pa[4] = {ua.x, ua.y, ua.z, ua.w}, pb[4] = {ub.x, ub.y, ub.z, ub.w};
    uint32_t r[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pa[j]));
      const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pb[j]));
      r[j] = pack_bf16x2(fmaf(wa, x.x, wb * y.x), fmaf(wa, x.y, wb * y.y));
    }
    __syncwarp();  // every lane of the row has read lse_a / lse_b before either is overwritten (in place)
    *reinterpret_cast<uint4*>(o + oi) = make_uint4(r[0], r[1], r[2], r[3]);
    if (c == 0) lse[li] = m + __logf(ea + eb);
  }
}

cudaError_t launch_lse_merge(const void* oa, const float* la, const void* ob, const float* lb, void* o, float* lse,
                             int B, int H, int N, int D, int num_sms, cudaStream_t stream) {
  const long long n = static_cast<long long>(B) * N * H * (D / 8);
  const long long blocks = (n + 255) / 256;
  const int grid = static_cast<int>(blocks < 16LL * num_sms ? blocks : 16LL * num_sms);
  const auto* a = static_cast<const __nv_bfloat16*>(oa);
  const auto* bb = static_cast<const __nv_bfloat16*>(ob);
  auto* out = static_cast<__nv_bfloat16*>(o);
  if (D == 64)
    s2_lse_merge_kernel<64><<<grid, 256, 0, stream>>>(a, la, bb, lb, out, lse, B, H, N);
  else
    s2_lse_merge_kernel<128><<<grid, 256, 0, stream>>>(a, la, bb, lb, out, lse, B, H, N);
  return cudaGetLastError();
}

}  // namespace s2
