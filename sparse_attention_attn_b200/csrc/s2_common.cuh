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
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace s2 {

constexpr int kTile = 128;  // rows of every q / kv tile
constexpr int kSub = 64;    // rows of a streamed backward sub-tile

struct Dims {
  int B, H, Hkv, N, D, G;
  int rep;        // H / Hkv, query heads per kv-head
  int n_groups;   // N / G
  int tiles;      // G / 128, tiles per group
  // Segment mode (chunk-wise attention over detached earlier keys): the key
  // tensors hold Nk rows and the N query rows sit at key position
  // qoff_t * 128 onwards; causal = 1: query row i sees keys [0, qoff_t*128 + i],
  // causal = 0: every key.  S2 attention: Nk = N, qoff_t = 0, causal = 1.
  int Nk, qoff_t, causal;
  // HGA block-sparse mode: no head is shifted, and every 256-row query block
  // also attends the historical 128-row key tiles listed for it (see HgaList)
  int noshift;
};

// Historical key tiles selected per 256-row query block (HGA digest: each
// query block loads a bounded set of exact historical tokens): int32
// [B, N/256, S] tile indices.  A block uses its leading entries that name a
// tile of an earlier segment (0 <= e < segment start / 128); the first entry
// outside that range ends the list.  null: no history.
struct HgaList {
  const int* tiles = nullptr;
  int S = 0;
};

constexpr int kQBlock = 256;  // query rows sharing one historical list

// Number of historical tiles query block qb (in segment g) attends; *list
// points at its entries.
__host__ __device__ __forceinline__ int hga_count(const Dims& d, const HgaList& hl, int b, int g, int qb,
                                                  const int** list) {
  *list = nullptr;
  if (hl.tiles == nullptr || hl.S <= 0) return 0;
  const int* l = hl.tiles + (static_cast<size_t>(b) * (d.N / kQBlock) + qb) * hl.S;
  const int lim = g * d.G / kTile;
  int n = 0;
  while (n < hl.S && l[n] >= 0 && l[n] < lim) ++n;
  *list = l;
  return n;
}

__host__ __device__ __forceinline__ int shift_of_head(const Dims& d, int h) {
  return (d.G < d.N && h >= d.H / 2 && !d.noshift) ? d.G / 2 : 0;
}

// Original row of rolled row r for a head with shift s.
__host__ __device__ __forceinline__ int original_row(const Dims& d, int r, int s) {
  int t = r + s;
  return t >= d.N ? t - d.N : t;
}

// Key row of rolled key row r for a head with shift s (the key tensors hold Nk rows).
__host__ __device__ __forceinline__ int original_row_kv(const Dims& d, int r, int s) {
  int t = r + s;
  return t >= d.Nk ? t - d.Nk : t;
}

// A work item: one 128-row tile of one rolled group of one (batch, head).
struct TileWork {
  int b, h, kvh, g, tile;  // tile = local tile index inside the group
};

// Persistent schedule.  A "unit" is one rolled group of one (batch, head);
// its T tiles are the work items.  Work grows (forward, dQ) or shrinks (dK/dV)
// linearly with the tile index, so tile t is paired with tile T-1-t: every
// pair carries the same work.  Pairs are dealt round-robin to the CTAs (one
// per SM), consecutive pairs belong to the same unit, so the CTAs running at
// one time share their K/V (or Q/dO) in L2.
// A launch can take a contiguous range [p0, pairs) of the pairs (the chunks
// of the split-dS backward); p0 = 0 and pairs = units * ppu otherwise.
struct PairSched {
  int units, T, ppu, pairs;  // ppu = pairs per unit; pairs = end of this launch's range
  int p0;                    // first pair of this launch's range
};

__host__ __device__ __forceinline__ PairSched make_pair_sched(int units, int T) {
  PairSched ps;
  ps.units = units;
  ps.T = T;
  ps.ppu = (T + 1) / 2;
  ps.pairs = units * ps.ppu;
  ps.p0 = 0;
  return ps;
}

// CTAs of a persistent launch over the range: one per pair, at most one per SM.
__host__ __device__ __forceinline__ int pair_grid(const PairSched& ps, int num_sms) {
  const int n = ps.pairs - ps.p0;
  return n < num_sms ? n : num_sms;
}

// Item `e` (0 or 1) of pair p: its unit and tile; false if it does not exist
// (the middle tile of an odd T has no partner).
__host__ __device__ __forceinline__ bool pair_item(const PairSched& ps, int p, int e, int& unit,
                                                   int& tile) {
  if (p >= ps.pairs) return false;
  unit = p / ps.ppu;
  const int pj = p - unit * ps.ppu;
  tile = (e == 0) ? pj : ps.T - 1 - pj;
  return !(e == 1 && tile == pj);
}

// Walks the items of one CTA in order: pairs p0 + blockIdx.x, +gridDim.x, ...
struct ItemCursor {
  int p, e, unit, tile, n;  // n = items visited before this one
  bool valid;
  __device__ __forceinline__ void first(const PairSched& ps) {
    p = ps.p0 + blockIdx.x;
    e = 0;
    n = 0;
    valid = pair_item(ps, p, e, unit, tile);
  }
  __device__ __forceinline__ void next(const PairSched& ps) {
    ++n;
    for (;;) {
      if (e == 0) {
        e = 1;
      } else {
        e = 0;
        p += gridDim.x;
      }
      if (p >= ps.pairs) {
        valid = false;
        return;
      }
      if (pair_item(ps, p, e, unit, tile)) {
        valid = true;
        return;
      }
    }
  }
};

// kv-tile work item of the dK/dV kernel from (unit, tile): unit = (b*Hkv + kvh)*ng + g.
__host__ __device__ __forceinline__ TileWork kv_item(const Dims& d, int unit, int tile) {
  TileWork w;
  w.tile = tile;
  w.g = unit % d.n_groups;
  const int x = unit / d.n_groups;
  w.kvh = x % d.Hkv;
  w.b = x / d.Hkv;
  w.h = w.kvh * d.rep;
  return w;
}

// query-tile work item of the forward / dQ kernels: unit = ((b*Hkv + kvh)*ng + g)*rep + hr.
__host__ __device__ __forceinline__ TileWork q_item(const Dims& d, int unit, int tile) {
  TileWork w;
  w.tile = tile;
  const int hr = unit % d.rep;
  int x = unit / d.rep;
  w.g = x % d.n_groups;
  x /= d.n_groups;
  w.kvh = x % d.Hkv;
  w.b = x / d.Hkv;
  w.h = w.kvh * d.rep + hr;
  return w;
}

// Sub-tile cursor of the dK/dV kernel: item (kv tile) plus sub-tile index.
struct DkvCursor {
  ItemCursor ic;
  TileWork w;
  int it, iters, nq;
  __device__ __forceinline__ void load(const Dims& d, const PairSched& ps) {
    if (!ic.valid) return;
    w = kv_item(d, ic.unit, ic.tile);
    nq = 2 * (d.tiles - w.tile);  // 64-row query sub-tiles from the diagonal to the group end
    iters = d.rep * nq;
    it = 0;
  }
  __device__ __forceinline__ void first(const Dims& d, const PairSched& ps) {
    ic.first(ps);
    load(d, ps);
  }
  __device__ __forceinline__ void next(const Dims& d, const PairSched& ps) {
    if (++it < iters) return;
    ic.next(ps);
    load(d, ps);
  }
};

// Forward schedule.  A forward item is a pair of adjacent query tiles
// (2i, 2i+1) of one unit (a rolled group of one (batch, head)): every K/V tile
// the first tile needs, the second needs too, so one K/V load feeds 256 query
// rows.  Item i carries 4i+3 tile products (2i+1 for the first tile, 2i+2 for
// the second).  Two static orders, chosen per shape by the host:
//  * snake: items sorted longest first, level-major (every unit's item Ti-1,
//    then every unit's Ti-2, ...), dealt boustrophedon over the CTAs.  This
//    approximates longest-processing-time-first list scheduling (within 3% of
//    perfect balance on the shapes served); CTAs running at one time work on
//    many units, so it is used when K and V together fit in L2;
//  * pairs: item i paired with item Ti-1-i (equal work), pairs dealt
//    round-robin, consecutive pairs in the same unit, so the CTAs running at
//    one time share their K/V in L2 (long sequences).
struct FwdSched {
  int snake;  // 1: snake order, 0: pairs
  int units;  // B * H * n_groups
  int Ti;     // items per unit, ceil(tiles / 2)
  int ppu;    // pairs per unit, ceil(Ti / 2)
  int n;      // snake: units * Ti items; pairs: units * ppu pairs
};

// The items of one CTA, in order.
struct FwdCursor {
  int r, e;     // round, and position inside the round
  int unit, i;  // current item
  bool valid;
  __device__ __forceinline__ void first(const FwdSched& s) {
    r = 0;
    e = 0;
    settle(s);
  }
  __device__ __forceinline__ void next(const FwdSched& s) {
    if (e == 0) {
      e = 1;
    } else {
      e = 0;
      ++r;
    }
    settle(s);
  }
  __device__ __forceinline__ void settle(const FwdSched& s) {
    const int P = gridDim.x, c = blockIdx.x;
    for (;;) {
      if (s.snake) {
        const int k = r * 2 * P + (e ? 2 * P - 1 - c : c);
        valid = k < s.n;  // positions only grow from here on
        if (valid) {
          const int lvl = k / s.units;
          unit = k - lvl * s.units;
          i = s.Ti - 1 - lvl;
        }
        return;
      }
      const int p = r * P + c;
      if (p >= s.n) {
        valid = false;
        return;
      }
      unit = p / s.ppu;
      const int pj = p - unit * s.ppu;
      i = e ? s.Ti - 1 - pj : pj;
      if (!(e && i == pj)) {
        valid = true;
        return;
      }
      e = 0;  // the middle item of an odd Ti has no partner
      ++r;
    }
  }
};

// One forward item: query tiles ta = 2i (always) and ta + 1 (if it exists),
// key/value tiles 0 .. nkv-1 of the same rolled group; lastA / lastB: the
// last key tile of tile A / B (its diagonal when causal), -1 if no tile B.
struct FwdItem {
  int b, h, kvh, g, sh;
  int ta;
  bool has_b;
  int nkv;
  int lastA, lastB;
  int nh;          // historical tiles first (HGA mode): key tile j < nh is hist[j]
  const int* hist;
};

__device__ __forceinline__ FwdItem fwd_item(const Dims& d, int unit, int i, const HgaList& hl) {
  const TileWork w = q_item(d, unit, 2 * i);
  FwdItem it;
  it.b = w.b;
  it.h = w.h;
  it.kvh = w.kvh;
  it.g = w.g;
  it.sh = shift_of_head(d, w.h);
  it.ta = 2 * i;
  it.has_b = 2 * i + 1 < d.tiles;
  it.nh = hga_count(d, hl, w.b, w.g, (w.g * d.G + it.ta * kTile) / kQBlock, &it.hist);
  const int nkt = d.Nk / kTile;
  const int off = d.qoff_t + it.nh;
  it.lastA = d.causal ? it.ta + off : nkt - 1;
  it.lastB = it.has_b ? (d.causal ? it.ta + 1 + off : nkt - 1) : -1;
  it.nkv = (it.has_b ? it.lastB : it.lastA) + 1;
  return it;
}

struct FwdArgs {
  Dims d;
  HgaList hist;            // HGA mode's historical tile lists (tiles = null otherwise)
  FwdSched sched;
  float scale_log2;        // (1/sqrt(D)) * log2(e)
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
  float* dqacc;            // fp32 [B, H, N, D] dQ accumulator zeroed here, or null (split path)
  uint32_t* status;        // device status words, cleared here (first kernel of the call)
};

struct BwdArgs {
  Dims d;
  HgaList hist;            // HGA mode (split path): historical tile lists for the dQ kernel
  PairSched kv_sched;      // dK/dV work items (units: batch x kv-head x group)
  PairSched q_sched;       // dQ work items (units: batch x head x group)
  float scale;             // 1/sqrt(D)
  float scale_log2;        // scale * log2(e)
  const float* ndelta;     // fp32 [B, H, N]: -Delta
  const float* nlse2;      // fp32 [B, H, N]: -lse * log2(e)
  void* dq;                // bf16 [B, N, H, D]
  int dq_accumulate;       // split path: dq += the result instead of dq = (segment pieces)
  int no_dkdv;             // split path: skip dK / dV (a detached key segment: dq only)
  float* dqacc;            // fused path: fp32 [B, H, N, D] dQ accumulator (zeroed by the preprocess)
  void* dk;                // bf16 [B, N, Hkv, D]
  void* dv;                // bf16 [B, N, Hkv, D]
  int kv_v8;               // dk and dv are 32-byte aligned: whole-sector stores
  const float* rope;       // fused path: fp32 (cos, sin) [N][D/2][2] table to rotate dq and dk back
                           // (the inputs were rotated by it), or null
  __nv_bfloat16* ds;       // split-dS path: the dK/dV kernel stores dS blocks here (see ds_block), or null
  int ds_tt;               // dS blocks per (batch, head, group): T (T + 1) / 2
  int ds_slots;            // dK/dV units whose dS the workspace holds at once (unit u uses slot u mod ds_slots)
  int kv_q128;             // dK/dV with 128-query tiles (s2_bwd_kv128.cu) instead of 64-query sub-tiles
  long long ds_blocks;     // dS blocks in all: ds_slots * rep * ds_tt
  uint32_t* status;
  unsigned long long wait_limit_ns;
};

// Split-dS path: index of the 128 x 128 dS block of (query tile i, kv tile
// j <= i) of group g of (batch b, query head h).  The blocks of one dK/dV unit
// u = (b Hkv + kvh) n_groups + g (its rep query heads) sit together in slot
// u mod slots; the workspace holds `slots` units at once, and the backward
// runs in pair ranges whose live units never share a slot.  A block holds dS^T
// as four slabs of 32 query columns, each [128 kv rows][32 queries] (64-byte
// rows).
__host__ __device__ __forceinline__ long long ds_block(const Dims& d, int b, int h, int g, int i, int j, int tt,
                                                       int slots) {
  const int kvh = h / d.rep;
  const int u = (b * d.Hkv + kvh) * d.n_groups + g;
  return (static_cast<long long>(u % slots) * d.rep + (h - kvh * d.rep)) * tt + i * (i + 1) / 2 + j;
}

// Split-dS path: pairs of dK/dV work per launch when the workspace holds
// `slots` units of dS (every unit: no chunking).  A range of c pairs starting
// anywhere touches at most 1 + ceil((c - 1) / ppu) units, which must fit the
// slots: c <= (slots - 1) ppu + 1.  Within that, whole rounds of `num_sms`
// pairs, so every launch but the last keeps all CTAs busy to its end.
__host__ __device__ __forceinline__ int ds_chunk_pairs(const PairSched& kv, int slots, int num_sms) {
  if (slots >= kv.units) return kv.pairs;
  const int maxc = (slots - 1) * kv.ppu + 1;
  return maxc >= num_sms ? maxc / num_sms * num_sms : maxc;
}

// TMA descriptors of the backward: 128-row and 64-row boxes of each operand.
struct BwdMaps {
  CUtensorMap q128, k128, v128, g128;
  CUtensorMap q64, k64, v64, g64;
  CUtensorMap ds, dq32;  // split-dS path: the dS blocks (2-D, 32 x 256 boxes), dq (32-row boxes)
};

template <int D>
cudaError_t launch_bwd_pre(const BwdPreArgs& pre, int num_sms, cudaStream_t stream);
// dK/dV with 128-query tiles: one launch over a.kv_sched's pair range.
template <int D>
cudaError_t launch_dkdv128(const BwdMaps& m, const BwdArgs& a, int num_sms, cudaStream_t stream);
template <int D>
cudaError_t launch_dq_ds(const CUtensorMap& tds, const CUtensorMap& tk, const CUtensorMap& tq32, const BwdArgs& a,
                         int num_sms, cudaStream_t stream);

// Index checks of the debug build (compiled with -DS2ATTN_DEBUG_CHECKS; they
// compile to nothing otherwise).  A computed global index outside [0, n)
// records status code 7 (S2ATTN_ERR_DEVICE_BOUNDS in the C ABI) and the site
// in the device status word pair -- the first failure wins -- and the caller
// skips the access.
constexpr uint32_t kDevBounds = 7;
__device__ __forceinline__ bool in_bounds(uint32_t* status, long long idx, long long n, uint32_t where) {
#ifdef S2ATTN_DEBUG_CHECKS
  if (idx >= 0 && idx < n) return true;
  if (status != nullptr && atomicCAS(status, 0u, kDevBounds) == 0u) status[1] = where;
  return false;
#else
  (void)status;
  (void)idx;
  (void)n;
  (void)where;
  return true;
#endif
}

// The 16 NF4 levels, ascending (index = 4-bit code), passed to the NF4 kernels.
struct Nf4Levels {
  float v[16];
};

// Arguments of the fused NF4 QKV projection kernel (s2_nf4.cu).
struct Nf4Args {
  const int8_t* sq;
  const float* c2;
  int width0, width1;  // features of q and of k (v has as many as k)
  int M, K;
  int tiles_w;  // 128-row weight tiles (Nout / 128)
  int tiles_t;  // 256-token tiles
  Nf4Levels lv;
  uint32_t* status;
  unsigned long long wait_limit_ns;
};

cudaError_t launch_nf4_qkv(const CUtensorMap& tx, const CUtensorMap& tc, const CUtensorMap* to, const Nf4Args& a,
                           int num_sms, cudaStream_t stream, int stages, int dq_warps);
cudaError_t launch_nf4_dequant(const void* codes, const int8_t* sq, const float* c2, void* w, long long n_words,
                               const Nf4Levels& lv, int num_sms, cudaStream_t stream);

// Optional per-kernel timing (s2attn_profile_start / _stop): the launchers
// bracket every kernel with these; they do nothing unless profiling is on.
enum KernelId : int {
  kKernelFwd = 0,
  kKernelBwdPre = 1,
  kKernelBwdDkDv = 2,
  kKernelBwdDq = 3,
  kKernelBwdFused = 4,
  kKernelBwdDqPost = 5,
  kKernelRope = 6,
  kKernelNf4Qkv = 7,
  kKernelNf4Dequant = 8,
  kKernelBwdDqDs = 9
};
void prof_before(cudaStream_t stream, int kernel_id);
void prof_after(cudaStream_t stream);

}  // namespace s2
