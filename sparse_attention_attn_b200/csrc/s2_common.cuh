// Shared definitions of the S2-Attn kernels: launch parameters, the shift /
// group index map and the work orderings.
//
// Index map (LongQLoRA community post, section 03, Shift Short Attention; the
// shifted half of the heads and the G/2 roll with wrap-around follow the
// LongLoRA method): query head h has shift s_h = G/2 if G < N and h >= H/2,
// else 0.  Rolled row r holds original row (r + s_h) mod N, rolled group
// r / G.  Because G/2 and N are multiples of the 128-row tile, a rolled tile
// [r0, r0 + 128) is the contiguous original range starting at (r0 + s_h) mod N,
// so the roll is folded into the TMA row coordinate and into the rows the
// epilogue stores: no rolled copy of any tensor exists.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace s2 {

constexpr int kTile = 128;  // rows of every q / kv tile

struct Dims {
  int B, H, Hkv, N, D, G;
  int rep;        // H / Hkv, query heads per kv-head
  int n_groups;   // N / G
  int tiles;      // G / 128, tiles per group
};

__host__ __device__ __forceinline__ int shift_of_head(const Dims& d, int h) {
  return (d.G < d.N && h >= d.H / 2) ? d.G / 2 : 0;
}

// Original row of rolled row r for a head with shift s.
__host__ __device__ __forceinline__ int original_row(const Dims& d, int r, int s) {
  int t = r + s;
  return t >= d.N ? t - d.N : t;
}

// Work item of one CTA.  Orders are unit-major so the CTAs resident at one time
// share their K/V (or Q/dO) tiles in L2, and longest-first inside a unit.
struct TileWork {
  int b, h, kvh, g, tile;  // tile = local tile index inside the group
};

// forward / dQ: one 128-row query tile of head h; work grows with the tile index.
__host__ __device__ __forceinline__ TileWork decode_q_tile(const Dims& d, int x) {
  TileWork w;
  const int T = d.tiles;
  w.tile = T - 1 - x % T;
  x /= T;
  const int hr = x % d.rep;
  x /= d.rep;
  w.g = x % d.n_groups;
  x /= d.n_groups;
  w.kvh = x % d.Hkv;
  w.b = x / d.Hkv;
  w.h = w.kvh * d.rep + hr;
  return w;
}

// dK/dV: one 128-row kv tile of kv-head kvh; work shrinks with the tile index.
__host__ __device__ __forceinline__ TileWork decode_kv_tile(const Dims& d, int x) {
  TileWork w;
  const int T = d.tiles;
  w.tile = x % T;
  x /= T;
  w.g = x % d.n_groups;
  x /= d.n_groups;
  w.kvh = x % d.Hkv;
  w.b = x / d.Hkv;
  w.h = w.kvh * d.rep;  // first query head of the kv-head (they share one shift)
  return w;
}

struct FwdArgs {
  Dims d;
  float scale_log2;        // (1/sqrt(D)) * log2(e)
  void* o;                 // bf16 [B, N, H, D]
  float* lse;              // fp32 [B, H, N]
  uint32_t* status;        // device status words
  unsigned long long wait_limit_ns;
};

struct BwdPreArgs {
  Dims d;
  const void* o;           // bf16 [B, N, H, D]
  const void* dO;          // bf16 [B, N, H, D]
  const float* lse;        // fp32 [B, H, N]
  float* ndelta;           // fp32 [B, H, N]: -Delta = -sum_d dO * O
  float* nlse2;            // fp32 [B, H, N]: -lse * log2(e)
  uint32_t* status;        // device status words, cleared here (first kernel of the call)
};

struct BwdArgs {
  Dims d;
  float scale;             // 1/sqrt(D)
  float scale_log2;        // scale * log2(e)
  const float* ndelta;     // fp32 [B, H, N]: -Delta
  const float* nlse2;      // fp32 [B, H, N]: -lse * log2(e)
  void* dq;                // bf16 [B, N, H, D]
  void* dk;                // bf16 [B, N, Hkv, D]
  void* dv;                // bf16 [B, N, Hkv, D]
  uint32_t* status;
  unsigned long long wait_limit_ns;
};

// TMA descriptors of the backward: 128-row and 64-row boxes of each operand.
struct BwdMaps {
  CUtensorMap q128, k128, v128, g128;
  CUtensorMap q64, k64, v64, g64;
};

// Optional per-kernel timing (s2attn_profile_start / _stop): the launchers
// bracket every kernel with these; they do nothing unless profiling is on.
enum KernelId : int { kKernelFwd = 0, kKernelBwdPre = 1, kKernelBwdDkDv = 2, kKernelBwdDq = 3 };
void prof_before(cudaStream_t stream, int kernel_id);
void prof_after(cudaStream_t stream);

}  // namespace s2
