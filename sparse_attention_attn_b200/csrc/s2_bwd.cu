// S2-Attn backward for sm_100a.
//
// Analytic gradient of softmax attention inside each rolled group, with P
// recomputed from the saved log-sum-exp (LongQLoRA community post, section 03,
// Shift Short Attention, used in training; the gradient formulas are those of
// plain softmax attention):
//   dP = dO V^T,  Delta_i = sum_d dO_id O_id,  dS = P * (dP - Delta),
//   dQ = scale dS K,  dK = scale dS^T Q,  dV = P^T dO.
//
// Three kernels run in order on one stream:
//   s2_bwd_pre_kernel   -Delta and -lse*log2(e) per query row (HBM-bound); stored
//                       negated so each score needs one fused multiply-add.
//   s2_bwd_dkdv_kernel  persistent; per 128-row kv tile of a kv-head it loops over
//                       the kv-head's query heads and the query sub-tiles from
//                       the diagonal to the end of the group.  S^T = K Q^T and
//                       dP^T = V dO^T land in TMEM, P^T and dS^T (bf16) are
//                       written back over them and feed dV += P^T dO and
//                       dK += dS^T Q straight from TMEM; dK/dV accumulate in
//                       TMEM for the whole loop (no atomics).
//   s2_bwd_dq_kernel    persistent; per 128-row query tile it loops over the kv
//                       sub-tiles from the group start to the diagonal: S, dP
//                       in TMEM, dS over dP, dQ += dS K in TMEM.
//
// Warp roles of the two UMMA kernels: warp 0 TMA producer, warp 1 TMEM owner
// and UMMA issuer, warps 2..9 elementwise and epilogue (thread = one TMEM lane
// = one tile row; warps 2..5 take the first 32 columns of each 64-column
// sub-tile and the first D/2 output columns, warps 6..9 the rest), and more
// UMMA issuers after them: warp 10 in dK/dV (352 threads), warps 10 and 11 in
// dQ (384 threads).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "s2_common.cuh"
#include "s2_ptx.cuh"

namespace s2 {

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ uint4 ldg_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ float dot_bf16x2(uint32_t a, uint32_t b) {
  const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&a));
  const float2 fb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&b));
  return fmaf(fa.x, fb.x, fa.y * fb.y);
}

// ------------------------------------------------------------------ preprocess

// One block per task of 128 consecutive rows t of one (batch, head): every
// row's D values are read as 16-byte chunks by D/8 lanes (whole rows per
// instruction), all of the task's loads are in flight at once, and the 128
// row statistics go out as contiguous runs through shared memory.
template <int D>
__global__ void __launch_bounds__(256) s2_bwd_pre_kernel(const BwdPreArgs a) {
  constexpr int LPR = D / 8;               // lanes per row: one 16-byte chunk each
  constexpr int RPS = 256 / LPR;           // rows per step (whole block)
  constexpr int STEPS = kTile / RPS;       // steps per 128-row task
  __shared__ float red[kTile];
  const Dims& d = a.d;
  const int tid = threadIdx.x;
  const int part = tid % LPR, rsub = tid / LPR;
  const uint4* o = static_cast<const uint4*>(a.o);
  const uint4* g = static_cast<const uint4*>(a.dO);
  if (blockIdx.x == 0 && tid == 0) {
    a.status[0] = 0u;
    a.status[1] = 0u;
  }
  const int tblk = d.N / kTile;
  const long long tasks = static_cast<long long>(d.B) * d.H * tblk;
  for (long long task = blockIdx.x; task < tasks; task += gridDim.x) {
    const long long bh = task / tblk;  // b * H + h
    const int t0 = static_cast<int>(task - bh * tblk) * kTile;
    const int h = static_cast<int>(bh % d.H), b = static_cast<int>(bh / d.H);
    uint4 ov[STEPS], gv[STEPS];
#pragma unroll
    for (int st = 0; st < STEPS; ++st) {
      const long long row = (static_cast<long long>(b) * d.N + t0 + st * RPS + rsub) * d.H + h;
      ov[st] = ldg_stream(o + row * (D / 8) + part);
      gv[st] = ldg_stream(g + row * (D / 8) + part);
    }
#pragma unroll
    for (int st = 0; st < STEPS; ++st) {
      float acc = dot_bf16x2(ov[st].x, gv[st].x) + dot_bf16x2(ov[st].y, gv[st].y) +
                  dot_bf16x2(ov[st].z, gv[st].z) + dot_bf16x2(ov[st].w, gv[st].w);
#pragma unroll
      for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (part == 0) red[st * RPS + rsub] = acc;
    }
    if (a.dqacc != nullptr) {
      // the fused backward reduces dQ partials into these 128 rows: start at zero
      float4* z = reinterpret_cast<float4*>(a.dqacc + (static_cast<size_t>(bh) * d.N + t0) * D);
#pragma unroll
      for (int i = 0; i < kTile * D / 4 / 256; ++i) z[tid + i * 256] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();
    if (tid < kTile) {
      const size_t idx = static_cast<size_t>(bh) * d.N + t0 + tid;
      if (in_bounds(a.status, static_cast<long long>(idx), static_cast<long long>(d.B) * d.H * d.N, 43)) {
        a.ndelta[idx] = -red[tid];
        a.nlse2[idx] = -a.lse[idx] * kLog2e;
      }
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------ dK / dV
//
// Persistent: one CTA per SM walks its share of 128-row kv tiles (work items,
// see PairSched).  The query side of each item streams in 64-row sub-tiles.
// S^T and dP^T (128 kv rows x 64 query columns each) are double-buffered in
// TMEM, so the UMMAs of sub-tile g+1 run while warps 2..9 turn sub-tile g into
// P^T and dS^T; the buffers, the Q/dO stages and their barriers run on one
// sub-tile counter across items.  One K/V buffer: it is released once the
// item's last S^T and dP^T have completed, and the next item's K/V load runs
// under that item's last gradient UMMAs and its epilogue (the issuers issue
// an item's last dV/dK before they wait for the next item's K/V; measured as
// fast as a second K/V buffer).  TMEM: S^T [0,128) (two 64-column buffers), dP^T
// [128,256), dV [256, 256+D), dK [256+D, 256+2D); dV/dK are read out by the
// epilogue of an item before the next item's first gradient UMMA overwrites
// them (acc_full / acc_free handshake).

// A-operand column of k-step kk (16 rows of K) when a 64-wide bf16 operand was
// written by two warp halves at packed columns [0,16) and [32,48) of its
// 64-column TMEM buffer (each half stays inside the fp32 columns it read).
__device__ __forceinline__ uint32_t split_acol64(int kk) { return kk * 8 + (kk >= 2 ? 16 : 0); }

template <int D, int NST>
struct DkvCfg {
  static constexpr int STAGES = NST;
  // warps: 0 producer, 1 UMMA issuer A, 2..9 elementwise + epilogue, 10 UMMA issuer B
  static constexpr int KV_ATOM = kTile * 128;  // one 64-column slab of a 128-row tile
  static constexpr int Q_ATOM = kSub * 128;    // one 64-column slab of a 64-row tile
  static constexpr int KV_BYTES = kTile * D * 2;
  static constexpr int Q_BYTES = kSub * D * 2;
  static constexpr int OFF_KV = 0;  // [K, V] of the current item
  static constexpr int OFF_Q = 2 * KV_BYTES;
  static constexpr int OFF_DO = OFF_Q + STAGES * Q_BYTES;
  static constexpr int OFF_ROW = OFF_DO + STAGES * Q_BYTES;  // per stage: -lse2[64], -delta[64]
  static constexpr int SMEM_BYTES = OFF_ROW + STAGES * 512 + 1024;
  static_assert(SMEM_BYTES <= 232448 - 512, "shared memory");
  static constexpr uint32_t TM_S = 0, TM_DP = 128, TM_DV = 256, TM_DK = 256 + D;
  static constexpr int THREADS = 352;
};

template <int D, int NST>
__global__ void __launch_bounds__(352, 1)
    s2_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmG,
                       const BwdArgs a) {
  using C = DkvCfg<D, NST>;
  constexpr int ST = C::STAGES;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  // bar_s / bar_dp: S^T / dP^T of a sub-tile landed (issuers A / B);
  // empty, kv_empty, acc_full complete once both issuers committed.
  __shared__ __align__(8) uint64_t bar_kv, bar_kv_empty, bar_full[ST], bar_empty[ST], bar_s[2],
      bar_dp[2], bar_pds[2], bar_acc_full, bar_acc_free, bar_drain[2];
  __shared__ uint32_t tmem_slot;
  __shared__ uint32_t abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Dims& d = a.d;
  const PairSched& ps = a.kv_sched;
  WaitCtx wc{&abort_flag, a.status, a.wait_limit_ns};

  const uint32_t s0 = smem_u32(smem);
  const uint32_t sK = s0 + C::OFF_KV, sV = s0 + C::OFF_KV + C::KV_BYTES;
  auto sQ = [&](int s) { return s0 + C::OFF_Q + s * C::Q_BYTES; };
  auto sG = [&](int s) { return s0 + C::OFF_DO + s * C::Q_BYTES; };
  auto sRow = [&](int s) { return s0 + C::OFF_ROW + s * 512; };

  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar_kv), 1);
    mbar_init(smem_u32(&bar_kv_empty), 2);  // the last S^T and dP^T of an item (one commit per issuer)
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bar_s[i]), 1);
      mbar_init(smem_u32(&bar_dp[i]), 1);
      mbar_init(smem_u32(&bar_pds[i]), 8);  // one elected arrival per elementwise warp
      mbar_init(smem_u32(&bar_drain[i]), 1);
    }
    for (int s = 0; s < ST; ++s) {
      mbar_init(smem_u32(&bar_full[s]), 1);
      mbar_init(smem_u32(&bar_empty[s]), 2);
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
    // (whole warp converged; one elected lane issues the copies)
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
      if (ic.n >= 1 && !warp_wait(smem_u32(&bar_kv_empty), (ic.n - 1) & 1, wc, 109)) break;
      // the kv tiles of this kernel are the query segment's own keys, which sit
      // at key rows qoff_t*128 onwards (0 for S2 attention)
      const int tk0 = original_row_kv(d, d.qoff_t * kTile + w.g * d.G + w.tile * kTile, sh);
      if (elect_one()) {
        mbar_arrive_expect_tx(smem_u32(&bar_kv), 2 * C::KV_BYTES);
        for (int c = 0; c < D / 64; ++c) {
          tma_load_4d(sK + c * C::KV_ATOM, &tmK, smem_u32(&bar_kv), c * 64, w.kvh, tk0, w.b);
          tma_load_4d(sV + c * C::KV_ATOM, &tmV, smem_u32(&bar_kv), c * 64, w.kvh, tk0, w.b);
        }
      }
      __syncwarp();
      ++kv_issued;
      const int nq = 2 * (d.tiles - w.tile);
      const int iters = d.rep * nq;
      for (int it = 0; it < iters; ++it, ++gi) {
        const int s = gi % ST, f = gi / ST;
        if (f > 0 && !warp_wait(smem_u32(&bar_empty[s]), (f - 1) & 1, wc, 110)) {
          ok = false;
          break;
        }
        const int h = w.kvh * d.rep + it / nq;
        const int i64 = 2 * w.tile + it % nq;
        const int tq0 = original_row(d, w.g * d.G + i64 * kSub, sh);
        const uint32_t bar = smem_u32(&bar_full[s]);
        if (elect_one()) {
          mbar_arrive_expect_tx(bar, 2 * C::Q_BYTES + 512);
          for (int c = 0; c < D / 64; ++c) {
            tma_load_4d(sQ(s) + c * C::Q_ATOM, &tmQ, bar, c * 64, h, tq0, w.b);
            tma_load_4d(sG(s) + c * C::Q_ATOM, &tmG, bar, c * 64, h, tq0, w.b);
          }
          const size_t ro = (static_cast<size_t>(w.b) * d.H + h) * d.N + tq0;
          bulk_load(sRow(s), a.nlse2 + ro, 256, bar);
          bulk_load(sRow(s) + 256, a.ndelta + ro, 256, bar);
        }
        __syncwarp();
      }
    }
    if (*wc.abort && lane == 0) {
      // never leave copies in flight into shared memory: wait (bounded) for
      // the last fill of every stage and of the K/V buffer
      if (kv_issued > 0) drain_wait(smem_u32(&bar_kv), (kv_issued - 1) & 1);
      for (int s = 0; s < ST && s < gi; ++s) drain_wait(smem_u32(&bar_full[s]), ((gi - 1 - s) / ST) & 1);
    }
  } else if (warp == 1 || warp == 10) {
    // ------------------------------------------------------------ UMMA issuers
    // Two converged warps on different SM sub-partitions share the UMMA
    // issue: A (warp 1) S^T = K Q^T and dV += P^T dO, B (warp 10) dP^T = V dO^T
    // and dK += dS^T Q.  Each stream is in order on its own; they meet only at
    // the barriers above.  (One issuing warp could not keep the tensor pipe
    // fed while eight elementwise warps share its sub-partitions.)
    const bool A = (warp == 1);
    const uint32_t idS = make_idesc_bf16(128, kSub, 0, 0);  // S^T, dP^T
    const uint32_t idG = make_idesc_bf16(128, D, 0, 1);     // dV, dK
    // A: operand K / Q / dO, B: operand V / dO / Q
    const uint64_t dX0 = make_sdesc_sw128(A ? sK : sV, 16, 1024);                // K-major (A operand)
    const uint64_t dYk = make_sdesc_sw128(A ? sQ(0) : sG(0), 16, 1024);          // K-major (B of S^T / dP^T)
    const uint64_t dZm = make_sdesc_sw128(A ? sG(0) : sQ(0), C::Q_ATOM, 1024);   // MN-major (B of dV / dK)
    const uint32_t tm_sp = tmem + (A ? C::TM_S : C::TM_DP);
    const uint32_t tm_acc = tmem + (A ? C::TM_DV : C::TM_DK);
    const uint32_t bar_ready = smem_u32(A ? &bar_s[0] : &bar_dp[0]);
    // S^T / dP^T of sub-tile g (cursor c); after an item's last one, the K/V
    // buffer goes back to the producer once those UMMAs have completed
    auto issue_sp = [&](int g, const DkvCursor& c) {
      const int s = g % ST;
      const uint32_t bo = (g & 1) * kSub;
      const uint64_t dy = sdesc_advance(dYk, s * C::Q_BYTES);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ko = (kk >> 2) * C::KV_ATOM + (kk & 3) * 32;
          const uint32_t qo = (kk >> 2) * C::Q_ATOM + (kk & 3) * 32;
          umma_ss(tm_sp + bo, sdesc_advance(dX0, ko), sdesc_advance(dy, qo), idS, kk > 0);
        }
        umma_commit(bar_ready + (g & 1) * 8);
        if (c.it == c.iters - 1) umma_commit(smem_u32(&bar_kv_empty));
      }
      __syncwarp();
    };
    // make sub-tile g (cursor c) ready: its item's K/V and its Q/dO stage
    auto wait_inputs = [&](const DkvCursor& c, int g) -> bool {
      if (c.it == 0 && !warp_wait(smem_u32(&bar_kv), c.ic.n & 1, wc, 120)) return false;
      if (!warp_wait(smem_u32(&bar_full[g % ST]), (g / ST) & 1, wc, 121)) return false;
      tc_fence_after();
      return true;
    };
    DkvCursor cur, nxt;
    cur.first(d, ps);
    nxt = cur;
    nxt.next(d, ps);
    bool ok = true;
    if (cur.ic.valid) {
      ok = wait_inputs(cur, 0);
      if (ok) issue_sp(0, cur);
    }
    for (int g = 0; ok && cur.ic.valid; ++g) {
      // the next sub-tile's S^T / dP^T (its TMEM buffer's last readers were
      // issued before: in order), ahead of this sub-tile's gradients -- unless
      // it opens the next item, whose K/V arrive only after this item's last
      // S^T / dP^T: then after them, so the epilogue never waits for that load
      const bool nxt_new = nxt.ic.valid && nxt.it == 0;
      if (nxt.ic.valid && !nxt_new) {
        if (!wait_inputs(nxt, g + 1)) break;
        issue_sp(g + 1, nxt);
      }
      if (!warp_wait(smem_u32(&bar_pds[g & 1]), (g >> 1) & 1, wc, 123)) break;
      if (cur.it == 0 && cur.ic.n > 0 &&
          !warp_wait(smem_u32(&bar_acc_free), (cur.ic.n - 1) & 1, wc, 124))
        break;
      tc_fence_after();
      const int s = g % ST;
      const uint32_t bo = (g & 1) * kSub;
      const uint64_t dz = sdesc_advance(dZm, s * C::Q_BYTES);
      const bool last = (cur.it == cur.iters - 1);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < kSub / 16; ++kk)
          umma_ts(tm_acc, tm_sp + bo + split_acol64(kk), sdesc_advance(dz, kk * 2048), idG,
                  (cur.it > 0 || kk > 0));
        umma_commit(smem_u32(&bar_empty[s]));
        if (last) umma_commit(smem_u32(&bar_acc_full));
      }
      __syncwarp();
      if (nxt_new) {
        if (!wait_inputs(nxt, g + 1)) break;
        issue_sp(g + 1, nxt);
      }
      cur = nxt;
      nxt.next(d, ps);
    }
    if (elect_one()) {
      umma_commit(smem_u32(&bar_drain[A ? 0 : 1]));
      drain_wait(smem_u32(&bar_drain[A ? 0 : 1]), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ P^T, dS^T, epilogue
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = quarter * 32 + lane;  // kv row inside the tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float sl2 = a.scale_log2;
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    bool ok = true;
    DkvCursor cur;
    cur.first(d, ps);
    long long ds_base = 0;
    for (int g = 0; cur.ic.valid; ++g) {
      const int s = g % ST;
      const int qoff = (cur.it % cur.nq) * kSub;  // query sub-tile start minus kv tile start (rolled)
      const uint32_t bo = (g & 1) * kSub + half * 32;
      ok = warp_wait(smem_u32(&bar_full[s]), (g / ST) & 1, wc, 130) &&
           warp_wait(smem_u32(&bar_s[g & 1]), (g >> 1) & 1, wc, 131) &&
           warp_wait(smem_u32(&bar_dp[g & 1]), (g >> 1) & 1, wc, 133);
      if (!ok) break;
      tc_fence_after();
      // row statistics of the 64 query rows: -lse*log2e at +0, -Delta at +256 bytes
      const uint32_t l4 = sRow(s) + half * 128, d4 = l4 + 256;
      float4 lv[8], dv4[8];
#pragma unroll
      for (int c4 = 0; c4 < 8; ++c4) {
        lv[c4] = lds_f4(l4 + c4 * 16);
        dv4[c4] = lds_f4(d4 + c4 * 16);
      }
      uint32_t sr[32], dr[32];
      tmem_ld32(tmem + lane_off + C::TM_S + bo, sr);
      tmem_ld32(tmem + lane_off + C::TM_DP + bo, dr);
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
      if (qoff < kTile) {  // sub-tile overlaps the diagonal: query before key is masked
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if (qoff + half * 32 + c < row) p[c] = 0.f;
      }
      uint32_t pk[16], dk[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) pk[c] = pack_bf16x2(p[2 * c], p[2 * c + 1]);
      tmem_st16(tmem + lane_off + C::TM_S + bo, pk);
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
      tmem_st16(tmem + lane_off + C::TM_DP + bo, dk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar_pds[g & 1]));
      if (a.ds != nullptr) {
        // split-dS path: these 32 dS^T values (kv row `row`, query columns
        // half * 32 + [0, 32) of sub-tile i64) also go to their dS block, in
        // its 32-column slab 2 (i64 & 1) + half: the warp's 32 rows write
        // 2 KB of consecutive bytes.  Issued after the arrival, so the dK
        // UMMA never waits for them.  The item's first block (query head
        // kvh rep, tile 0, kv tile 0) is formed once per item; then query
        // head, query tile and kv tile as ds_block orders them.
        if (cur.it == 0) ds_base = ds_block(d, cur.w.b, cur.w.h, cur.w.g, 0, 0, a.ds_tt, a.ds_slots);
        const int i64 = 2 * cur.w.tile + cur.it % cur.nq, i = i64 >> 1;
        const long long blk = ds_base + static_cast<long long>(cur.it / cur.nq) * a.ds_tt + i * (i + 1) / 2 + cur.w.tile;
        if (in_bounds(wc.status, blk, a.ds_blocks, 48)) {
          __nv_bfloat16* dst = a.ds + blk * (kTile * kTile) + (2 * (i64 & 1) + half) * (kTile * 32) + row * 32;
          const uint32_t lo[8] = {dk[0], dk[1], dk[2], dk[3], dk[4], dk[5], dk[6], dk[7]};
          const uint32_t hi[8] = {dk[8], dk[9], dk[10], dk[11], dk[12], dk[13], dk[14], dk[15]};
          st_global_v8(dst, lo);
          st_global_v8(dst + 16, hi);
        }
      }
      if (cur.it == cur.iters - 1) {
        // ---------------------------------------------------- epilogue of this item
        ok = warp_wait(smem_u32(&bar_acc_full), cur.ic.n & 1, wc, 132);
        if (!ok) break;
        tc_fence_after();
        const TileWork& w = cur.w;
        const int tk0 = original_row(d, w.g * d.G + w.tile * kTile, shift_of_head(d, w.h));
        const size_t grow = (static_cast<size_t>(w.b) * d.N + tk0 + row) * d.Hkv + w.kvh;
        const bool grow_ok =
            in_bounds(wc.status, static_cast<long long>(grow), static_cast<long long>(d.B) * d.N * d.Hkv, 44);
        __nv_bfloat16* dvrow = static_cast<__nv_bfloat16*>(a.dv) + grow * D + half * (D / 2);
        __nv_bfloat16* dkrow = static_cast<__nv_bfloat16*>(a.dk) + grow * D + half * (D / 2);
        uint32_t r[D / 64][32], r2[D / 64][32];
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          tmem_ld32(tmem + lane_off + C::TM_DV + half * (D / 2) + c * 32, r[c]);
          tmem_ld32(tmem + lane_off + C::TM_DK + half * (D / 2) + c * 32, r2[c]);
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

// ------------------------------------------------------------------ dQ
//
// Persistent: one CTA per SM walks its share of 128-row query tiles.  Keys and
// values of each item stream in 64-row sub-tiles from the group start to the
// diagonal.  S and dP (128 x 64) are double-buffered in TMEM so the UMMAs of
// sub-tile g+1 overlap the dS work on sub-tile g.  Q / dO arrive by TMA in one
// shared-memory buffer and are copied, one item at a time, into TMEM by the dS
// warps, so S = Q K^T and dP = dO V^T take their A operand from TMEM and read
// only K / V from shared memory (an SS UMMA with N = 64 would be limited by
// shared-memory bandwidth); the buffer then takes the next item's Q / dO.
// Three UMMA issuers split the sub-tile's 20 instructions (next to busy
// elementwise warps one issuing thread spends far longer per UMMA than a TS
// UMMA with N = 64 executes): warp 1 issues S, warp 10 dP, warp 11
// dQ += dS K; warp 10 overwrites a dS buffer only after warp 11's dQ that
// read it has completed (bar_dqd).  The epilogue stages each
// warp's 32 rows of dQ in shared memory and writes them back row-contiguous.
// TMEM: S [0,128) (two buffers), dP [128,256), dQ [256, 256+D),
// Q [256+D, 256+3D/2), dO [256+3D/2, 256+2D) (bf16 pairs); dQ is read out by
// the item's epilogue before the next item overwrites it.

template <int D, int NST>
struct DqCfg {
  static constexpr int STAGES = NST;
  static constexpr int Q_ATOM = kTile * 128;
  static constexpr int KV_ATOM = kSub * 128;
  static constexpr int Q_BYTES = kTile * D * 2;
  static constexpr int KV_BYTES = kSub * D * 2;
  static constexpr int ROW_OUT = D;                 // bytes of one row's half of dQ (D/2 bf16)
  static constexpr int OFF_Q = 0;                   // [Q, dO]
  static constexpr int OFF_OUT = 2 * Q_BYTES;       // epilogue staging: 8 warps x 32 rows x ROW_OUT
  static constexpr int OFF_K = OFF_OUT + 8 * 32 * ROW_OUT;
  static constexpr int OFF_V = OFF_K + STAGES * KV_BYTES;
  static constexpr int SMEM_BYTES = OFF_V + STAGES * KV_BYTES + 1024;
  static constexpr uint32_t TM_S = 0, TM_DP = 128, TM_DQ = 256;
  static constexpr uint32_t TM_QT = 256 + D, TM_GT = 256 + D + D / 2;  // Q, dO as UMMA A operands
  static constexpr int THREADS = 384;
  static_assert(SMEM_BYTES <= 232448 - 512, "shared memory");
};

struct DqCursor {
  ItemCursor ic;
  TileWork w;
  int it, iters;
  int nh;            // HGA mode: the query block's historical tiles (64-row sub-tiles j < 2 nh)
  const int* hist;
  __device__ __forceinline__ void load(const Dims& d, const HgaList& hl) {
    if (!ic.valid) return;
    w = q_item(d, ic.unit, ic.tile);
    nh = hga_count(d, hl, w.b, w.g, (w.g * d.G + w.tile * kTile) / kQBlock, &hist);
    // 64-row kv sub-tiles: the listed historical tiles, then from the group
    // start to the diagonal (causal), or every key (segment mode, causal = 0)
    iters = d.causal ? 2 * (w.tile + 1 + d.qoff_t + nh) : 2 * (d.Nk / kTile);
    it = 0;
  }
  __device__ __forceinline__ void first(const Dims& d, const PairSched& ps, const HgaList& hl) {
    ic.first(ps);
    load(d, hl);
  }
  __device__ __forceinline__ void next(const Dims& d, const PairSched& ps, const HgaList& hl) {
    if (++it < iters) return;
    ic.next(ps);
    load(d, hl);
  }
  // key row of 64-row kv sub-tile j of this item
  __device__ __forceinline__ int kv_row(const Dims& d, int j) const {
    if (j < 2 * nh) return hist[j >> 1] * kTile + (j & 1) * kSub;
    return original_row_kv(d, w.g * d.G + (j - 2 * nh) * kSub, shift_of_head(d, w.h));
  }
};

template <int D, int NST>
__global__ void __launch_bounds__(384, 1)
    s2_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmG,
                     const BwdArgs a) {
  using C = DqCfg<D, NST>;
  constexpr int ST = C::STAGES;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ __align__(8) uint64_t bar_q, bar_q_empty, bar_qt, bar_kv[ST], bar_empty[ST], bar_sdp[2], bar_ds[2],
      bar_acc_full, bar_acc_free, bar_dqd[2], bar_drain[3];
  __shared__ uint32_t tmem_slot;
  __shared__ uint32_t abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Dims& d = a.d;
  const PairSched& ps = a.q_sched;
  WaitCtx wc{&abort_flag, a.status, a.wait_limit_ns};

  const uint32_t s0 = smem_u32(smem);
  const uint32_t sQ = s0 + C::OFF_Q, sG = s0 + C::OFF_Q + C::Q_BYTES;
  auto sK = [&](int s) { return s0 + C::OFF_K + s * C::KV_BYTES; };
  auto sV = [&](int s) { return s0 + C::OFF_V + s * C::KV_BYTES; };

  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar_q), 1);
    mbar_init(smem_u32(&bar_q_empty), 8);  // the dS warps, once Q / dO are in TMEM
    mbar_init(smem_u32(&bar_qt), 8);       // one elected arrival per dS warp
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bar_sdp[i]), 2);  // S (warp 1) and dP (warp 10)
      mbar_init(smem_u32(&bar_ds[i]), 8);   // one elected arrival per dS warp
      mbar_init(smem_u32(&bar_dqd[i]), 1);  // dQ(g) (warp 11) done with dS buffer g&1
    }
    for (int i = 0; i < 3; ++i) mbar_init(smem_u32(&bar_drain[i]), 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(smem_u32(&bar_kv[s]), 1);
      mbar_init(smem_u32(&bar_empty[s]), 1);
    }
    mbar_init(smem_u32(&bar_acc_full), 1);
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
    int gi = 0, q_issued = 0;
    bool ok = true;
    DqCursor pc;  // walks items only (it is left at 0)
    for (pc.first(d, ps, a.hist); ok && pc.ic.valid; pc.ic.next(ps), pc.load(d, a.hist)) {
      const ItemCursor& ic = pc.ic;
      const TileWork w = pc.w;
      const int sh = shift_of_head(d, w.h);
      // the buffer is free once the previous item's Q / dO are in TMEM
      if (ic.n >= 1 && !warp_wait(smem_u32(&bar_q_empty), (ic.n - 1) & 1, wc, 209)) break;
      const int tq0 = original_row(d, w.g * d.G + w.tile * kTile, sh);
      if (elect_one()) {
        mbar_arrive_expect_tx(smem_u32(&bar_q), 2 * C::Q_BYTES);
        for (int c = 0; c < D / 64; ++c) {
          tma_load_4d(sQ + c * C::Q_ATOM, &tmQ, smem_u32(&bar_q), c * 64, w.h, tq0, w.b);
          tma_load_4d(sG + c * C::Q_ATOM, &tmG, smem_u32(&bar_q), c * 64, w.h, tq0, w.b);
        }
      }
      __syncwarp();
      ++q_issued;
      const int iters = pc.iters;
      for (int j = 0; j < iters; ++j, ++gi) {
        const int s = gi % ST, f = gi / ST;
        if (f > 0 && !warp_wait(smem_u32(&bar_empty[s]), (f - 1) & 1, wc, 210)) {
          ok = false;
          break;
        }
        const int tk0 = pc.kv_row(d, j);
        const uint32_t bar = smem_u32(&bar_kv[s]);
        if (elect_one()) {
          mbar_arrive_expect_tx(bar, 2 * C::KV_BYTES);
          for (int c = 0; c < D / 64; ++c) {
            tma_load_4d(sK(s) + c * C::KV_ATOM, &tmK, bar, c * 64, w.kvh, tk0, w.b);
            tma_load_4d(sV(s) + c * C::KV_ATOM, &tmV, bar, c * 64, w.kvh, tk0, w.b);
          }
        }
        __syncwarp();
      }
    }
    if (*wc.abort && lane == 0) {
      if (q_issued > 0) drain_wait(smem_u32(&bar_q), (q_issued - 1) & 1);
      for (int s = 0; s < ST && s < gi; ++s) drain_wait(smem_u32(&bar_kv[s]), ((gi - 1 - s) / ST) & 1);
    }
  } else if (warp == 1 || warp >= 10) {
    // ------------------------------------------------------------ UMMA issuers
    // warp 1: S(g) = Q K_g^T.  warp 10: dP(g) = dO V_g^T.  warp 11:
    // dQ += dS(g) K_g.  S and dP wait for dS(g-2) before writing buffer g&1
    // again, dP also for dQ(g-2), the last reader of that dS buffer.
    const bool is_s = (warp == 1);
    const int role = (warp == 1) ? 0 : (warp == 10 ? 1 : 2);
    const uint32_t idS = make_idesc_bf16(128, kSub, 0, 0);  // S, dP: A from TMEM, B K-major
    const uint32_t idQ = make_idesc_bf16(128, D, 0, 1);     // dQ += dS K (K MN-major)
    const uint64_t dKk = make_sdesc_sw128(sK(0), 16, 1024);            // K-major (B of S)
    const uint64_t dVk = make_sdesc_sw128(sV(0), 16, 1024);            // K-major (B of dP)
    const uint64_t dKm = make_sdesc_sw128(sK(0), C::KV_ATOM, 1024);    // MN-major (B of dQ)
    const uint32_t tA = tmem + (is_s ? C::TM_QT : C::TM_GT);
    const uint32_t tD = tmem + (is_s ? C::TM_S : C::TM_DP);
    const uint64_t dB0 = is_s ? dKk : dVk;
    // S or dP of sub-tile g (cursor c)
    auto issue_sdp = [&](const DqCursor& c, int g) -> bool {
      if (c.it == 0 && !warp_wait(smem_u32(&bar_qt), c.ic.n & 1, wc, 220)) return false;
      if (!warp_wait(smem_u32(&bar_kv[g % ST]), (g / ST) & 1, wc, 221)) return false;
      if (g >= 2 && !warp_wait(smem_u32(&bar_ds[g & 1]), ((g - 2) >> 1) & 1, wc, 222)) return false;
      if (role == 1 && g >= 2 && !warp_wait(smem_u32(&bar_dqd[g & 1]), ((g - 2) >> 1) & 1, wc, 225)) return false;
      tc_fence_after();
      const uint64_t db = sdesc_advance(dB0, (g % ST) * C::KV_BYTES);
      const uint32_t bo = (g & 1) * kSub;
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ko = (kk >> 2) * C::KV_ATOM + (kk & 3) * 32;
          umma_ts(tD + bo, tA + kk * 8, sdesc_advance(db, ko), idS, kk > 0);
        }
        umma_commit(smem_u32(&bar_sdp[g & 1]));
      }
      __syncwarp();
      return true;
    };
    // dQ += dS(g) K_g (warp 10)
    auto issue_dq = [&](const DqCursor& c, int g) -> bool {
      if (!warp_wait(smem_u32(&bar_ds[g & 1]), (g >> 1) & 1, wc, 223)) return false;
      if (c.it == 0 && c.ic.n > 0 && !warp_wait(smem_u32(&bar_acc_free), (c.ic.n - 1) & 1, wc, 224))
        return false;
      tc_fence_after();
      const int s = g % ST;
      const uint32_t bo = (g & 1) * kSub;
      const uint64_t dk = sdesc_advance(dKm, s * C::KV_BYTES);
      const bool last = (c.it == c.iters - 1);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < kSub / 16; ++kk)
          umma_ts(tmem + C::TM_DQ, tmem + C::TM_DP + bo + split_acol64(kk), sdesc_advance(dk, kk * 2048), idQ,
                  (c.it > 0 || kk > 0));
        // S(g) and dP(g) have completed: the dS warps read them before dS(g)
        umma_commit(smem_u32(&bar_empty[s]));
        umma_commit(smem_u32(&bar_dqd[g & 1]));
        if (last) umma_commit(smem_u32(&bar_acc_full));
      }
      __syncwarp();
      return true;
    };
    DqCursor cur;
    cur.first(d, ps, a.hist);
    bool ok = true;
    for (int g = 0; ok && cur.ic.valid; ++g) {
      ok = (role == 2) ? issue_dq(cur, g) : issue_sdp(cur, g);
      cur.next(d, ps, a.hist);
    }
    // every issued UMMA completes before TMEM is released
    if (elect_one()) {
      umma_commit(smem_u32(&bar_drain[role]));
      drain_wait(smem_u32(&bar_drain[role]), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ dS, epilogue
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = quarter * 32 + lane;  // query row inside the tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint64_t sl2x2 = f2_pack(a.scale_log2, a.scale_log2);
    // this warp's epilogue staging: 32 rows x ROW_OUT bytes, 16-byte chunks
    // swizzled by the row so neither the row-wise writes nor the column-wise
    // reads conflict
    const uint32_t stage = s0 + C::OFF_OUT + (warp - 2) * 32 * C::ROW_OUT;
    constexpr int CH = C::ROW_OUT / 16;  // 16-byte chunks per staged row
    bool ok = true;
    uint64_t nl2 = 0, nd2 = 0;
    // Item c's Q rows (warps of half 0) or dO rows (half 1) from the swizzled
    // shared-memory tile into TMEM as bf16 pairs: the A operand of S / dP.
    // Called once the previous item's last S and dP have completed.
    auto put_q = [&](const DqCursor& c) -> bool {
      if (!warp_wait(smem_u32(&bar_q), c.ic.n & 1, wc, 233)) return false;
      const uint32_t src = (half == 0 ? sQ : sG) + row * 128;
      const uint32_t sw = static_cast<uint32_t>(row & 7);
#pragma unroll
      for (int at = 0; at < D / 64; ++at) {
        uint32_t r[32];
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const float4 v = lds_f4(src + at * C::Q_ATOM + ((ch ^ sw) << 4));
          r[4 * ch] = __float_as_uint(v.x);
          r[4 * ch + 1] = __float_as_uint(v.y);
          r[4 * ch + 2] = __float_as_uint(v.z);
          r[4 * ch + 3] = __float_as_uint(v.w);
        }
        tmem_st32(tmem + lane_off + (half == 0 ? C::TM_QT : C::TM_GT) + at * 32, r);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(&bar_qt));
        mbar_arrive(smem_u32(&bar_q_empty));  // the shared-memory copy may be overwritten
      }
      return true;
    };
    // this thread's row statistics of item c: -lse * log2 e and -Delta
    auto row_stats = [&](const DqCursor& c, float& l2, float& dl) {
      const TileWork& w = c.w;
      const int t0 = original_row(d, w.g * d.G + w.tile * kTile, shift_of_head(d, w.h));
      const size_t ridx = (static_cast<size_t>(w.b) * d.H + w.h) * d.N + t0 + row;
      l2 = 0.f;
      dl = 0.f;
      if (in_bounds(wc.status, static_cast<long long>(ridx), static_cast<long long>(d.B) * d.H * d.N, 45)) {
        l2 = a.nlse2[ridx];
        dl = a.ndelta[ridx];
      }
    };
    DqCursor cur;
    cur.first(d, ps, a.hist);
    float nl_next = 0.f, nd_next = 0.f;  // the next item's, fetched one item ahead
    if (cur.ic.valid) {
      ok = put_q(cur);
      row_stats(cur, nl_next, nd_next);
    }
    for (int g = 0; ok && cur.ic.valid; ++g) {
      const TileWork& w = cur.w;
      const int tq0 = original_row(d, w.g * d.G + w.tile * kTile, shift_of_head(d, w.h));
      if (cur.it == 0) {
        nl2 = f2_pack(nl_next, nl_next);
        nd2 = f2_pack(nd_next, nd_next);
      }
      const uint32_t bo = (g & 1) * kSub + half * 32;
      // kv sub-tile start minus query tile start (in the sub-tile walk: the
      // historical tiles and the segment offset come first)
      const int koff = cur.it * kSub - (w.tile + d.qoff_t + cur.nh) * kTile;
      ok = warp_wait(smem_u32(&bar_sdp[g & 1]), (g >> 1) & 1, wc, 230);
      if (!ok) break;
      tc_fence_after();
      if (cur.it == cur.iters - 1) {
        // this item's last S and dP are done with Q / dO in TMEM: bring in the
        // next item's, so its first S / dP overlap the dS work below
        DqCursor nq = cur;
        nq.next(d, ps, a.hist);
        if (nq.ic.valid) {
          if (!put_q(nq)) {
            ok = false;
            break;
          }
          row_stats(nq, nl_next, nd_next);  // in flight during this item's last dS and epilogue
        }
      }
      uint32_t sr[32], dr[32];
      tmem_ld32(tmem + lane_off + C::TM_S + bo, sr);
      tmem_ld32(tmem + lane_off + C::TM_DP + bo, dr);
      tmem_wait_ld();
      float p[32];
#pragma unroll
      for (int c = 0; c < 16; ++c) {  // P = 2^(S * scale * log2 e - lse * log2 e)
        const uint64_t x = f2_fma(f2_pack(__uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1])), sl2x2, nl2);
        p[2 * c] = ex2_approx(f2_lo(x));
        p[2 * c + 1] = ex2_approx(f2_hi(x));
      }
      if (d.causal && koff >= 0) {  // sub-tile overlaps the diagonal: key after query is masked
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if (koff + half * 32 + c > row) p[c] = 0.f;
      }
      uint32_t pk[16];
#pragma unroll
      for (int c = 0; c < 16; ++c)  // dS = P * (dP - Delta)
        pk[c] = f2_to_bf16x2(f2_mul(f2_pack(p[2 * c], p[2 * c + 1]),
                                    f2_add(f2_pack(__uint_as_float(dr[2 * c]), __uint_as_float(dr[2 * c + 1])), nd2)));
      tmem_st16(tmem + lane_off + C::TM_DP + bo, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar_ds[g & 1]));
      if (cur.it == cur.iters - 1) {
        // ---------------------------------------------------- epilogue of this item
        ok = warp_wait(smem_u32(&bar_acc_full), cur.ic.n & 1, wc, 232);
        if (!ok) break;
        tc_fence_after();
        // this thread's row, columns [half * D/2, (half+1) * D/2), scaled,
        // as bf16 into the staging rows
        const uint32_t srow = stage + lane * C::ROW_OUT;
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          uint32_t r[32];
          tmem_ld32(tmem + lane_off + C::TM_DQ + half * (D / 2) + c * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int ch = c * 4 + q;
            st_shared_v4(srow + ((ch ^ (lane % CH)) << 4),
                         pack_bf16x2(__uint_as_float(r[8 * q]) * a.scale, __uint_as_float(r[8 * q + 1]) * a.scale),
                         pack_bf16x2(__uint_as_float(r[8 * q + 2]) * a.scale, __uint_as_float(r[8 * q + 3]) * a.scale),
                         pack_bf16x2(__uint_as_float(r[8 * q + 4]) * a.scale, __uint_as_float(r[8 * q + 5]) * a.scale),
                         pack_bf16x2(__uint_as_float(r[8 * q + 6]) * a.scale, __uint_as_float(r[8 * q + 7]) * a.scale));
          }
        }
        // dQ is out of TMEM: the next item's first dQ UMMA may start
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bar_acc_free));
        // write back row-contiguous: lane l takes chunk l % CH of staged row
        // 32/CH * i + l / CH, so each store instruction covers whole rows
        __nv_bfloat16* dq0 = static_cast<__nv_bfloat16*>(a.dq) +
                             ((static_cast<size_t>(w.b) * d.N + tq0 + quarter * 32) * d.H + w.h) * D + half * (D / 2);
#pragma unroll
        for (int i = 0; i < CH; ++i) {
          const int rr = i * (32 / CH) + lane / CH, ch = lane % CH;
          float4 v = lds_f4(stage + rr * C::ROW_OUT + ((ch ^ (rr % CH)) << 4));
          const long long qrow = (static_cast<long long>(w.b) * d.N + tq0 + quarter * 32 + rr) * d.H + w.h;
          if (!in_bounds(wc.status, qrow, static_cast<long long>(d.B) * d.N * d.H, 46)) continue;
          float4* dst = reinterpret_cast<float4*>(dq0 + static_cast<size_t>(rr) * d.H * D + ch * 8);
          if (a.dq_accumulate) {  // dq += this piece (8 bf16 values, summed in fp32)
            const float4 old = *dst;
            const uint32_t* o32 = reinterpret_cast<const uint32_t*>(&old);
            uint32_t* n32 = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&o32[u]));
              const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&n32[u]));
              n32[u] = pack_bf16x2(x.x + y.x, x.y + y.y);
            }
          }
          *dst = v;
        }
        __syncwarp();
      }
      cur.next(d, ps, a.hist);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ launchers

static bool set_smem_attr(const void* fn, int bytes) {
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess;
}

// The preprocess: one block per 128-row task of one (batch, head), at most
// sixteen blocks per SM.
template <int D>
cudaError_t launch_bwd_pre(const BwdPreArgs& pre, int num_sms, cudaStream_t stream) {
  const long long rows = static_cast<long long>(pre.d.B) * pre.d.N * pre.d.H;
  const long long tasks = rows / kTile;  // 128-row tasks of one (batch, head)
  // up to 16 blocks per SM (8 resident at a time): blocks that finish early
  // take the remaining tasks (0.050 vs 0.054 ms at the Qwen3-8B shape with 8)
  const int pre_grid = static_cast<int>(tasks < 16LL * num_sms ? tasks : 16LL * num_sms);
  prof_before(stream, kKernelBwdPre);
  s2_bwd_pre_kernel<D><<<pre_grid, 256, 0, stream>>>(pre);
  cudaError_t e = cudaGetLastError();
  prof_after(stream);
  return e;
}
template cudaError_t launch_bwd_pre<64>(const BwdPreArgs&, int, cudaStream_t);
template cudaError_t launch_bwd_pre<128>(const BwdPreArgs&, int, cudaStream_t);

// Tensor maps: `*128` have 128-row boxes, `*64` 64-row boxes.  dK/dV streams
// 64-row query sub-tiles against 128-row kv tiles; dQ the other way round.
// NST: pipeline stages of the dK/dV kernel's streamed operands; the split
// path's dQ kernel takes the same, at most 3 at head dim 128 (what fits).
template <int D, int NST>
cudaError_t launch_bwd_stages(const BwdMaps& m, const BwdPreArgs& pre, const BwdArgs& a, int num_sms,
                              cudaStream_t stream, int* launches) {
  constexpr int QST = (D == 128 && NST > 3) ? 3 : NST;
  using K3 = DkvCfg<D, NST>;
  using K4 = DqCfg<D, QST>;
  if (!set_smem_attr(reinterpret_cast<const void*>(s2_bwd_dkdv_kernel<D, NST>), K3::SMEM_BYTES) ||
      !set_smem_attr(reinterpret_cast<const void*>(s2_bwd_dq_kernel<D, QST>), K4::SMEM_BYTES))
    return cudaErrorInvalidValue;
  cudaError_t e = launch_bwd_pre<D>(pre, num_sms, stream);
  if (e != cudaSuccess) return e;
  if (a.ds != nullptr) {
    // split-dS path: dK/dV over consecutive ranges of its pairs, each followed
    // by dQ for the units the range completed (their dS blocks all stored);
    // the workspace's slots then serve the next range's units.  One range
    // when every unit's dS fits.
    const int total = a.kv_sched.pairs, ppu = a.kv_sched.ppu;
    const int chunk = ds_chunk_pairs(a.kv_sched, a.ds_slots, num_sms);
    BwdArgs c = a;
    int done = 0, n = 1;
    for (int p0 = 0; p0 < total; p0 += chunk) {
      const int p1 = p0 + chunk < total ? p0 + chunk : total;
      c.kv_sched.p0 = p0;
      c.kv_sched.pairs = p1;
      if (a.kv_q128) {
        e = launch_dkdv128<D>(m, c, num_sms, stream);
      } else {
        prof_before(stream, kKernelBwdDkDv);
        s2_bwd_dkdv_kernel<D, NST><<<pair_grid(c.kv_sched, num_sms), K3::THREADS, K3::SMEM_BYTES, stream>>>(
            m.q64, m.k128, m.v128, m.g64, c);
        e = cudaGetLastError();
        prof_after(stream);
      }
      if (e != cudaSuccess) return e;
      ++n;
      const int upto = p1 / ppu;  // units with every pair done
      if (upto > done) {
        c.q_sched.p0 = done * a.d.rep * a.q_sched.ppu;
        c.q_sched.pairs = upto * a.d.rep * a.q_sched.ppu;
        e = launch_dq_ds<D>(m.ds, m.k128, m.dq32, c, num_sms, stream);
        if (e != cudaSuccess) return e;
        ++n;
        done = upto;
      }
    }
    if (launches) *launches = n;
    return cudaSuccess;
  }
  if (!a.no_dkdv && a.kv_q128) {
    e = launch_dkdv128<D>(m, a, num_sms, stream);
    if (e != cudaSuccess) return e;
  } else if (!a.no_dkdv) {
    const int grid_kv = pair_grid(a.kv_sched, num_sms);
    prof_before(stream, kKernelBwdDkDv);
    s2_bwd_dkdv_kernel<D, NST><<<grid_kv, K3::THREADS, K3::SMEM_BYTES, stream>>>(m.q64, m.k128, m.v128, m.g64, a);
    e = cudaGetLastError();
    prof_after(stream);
    if (e != cudaSuccess) return e;
  }
  if (launches) *launches = a.no_dkdv ? 2 : 3;
  const int grid_q = pair_grid(a.q_sched, num_sms);
  prof_before(stream, kKernelBwdDq);
  s2_bwd_dq_kernel<D, QST><<<grid_q, K4::THREADS, K4::SMEM_BYTES, stream>>>(m.q128, m.k64, m.v64, m.g128, a);
  e = cudaGetLastError();
  prof_after(stream);
  return e;
}

// stages: 2, 3 or 4 at head dim 128, 3 or 4 at head dim 64 (what fits in
// shared memory); anything else is an invalid value.
template <int D>
cudaError_t launch_bwd(const BwdMaps& m, const BwdPreArgs& pre, const BwdArgs& a, int num_sms,
                       cudaStream_t stream, int* launches, int stages) {
  if constexpr (D == 128) {
    if (stages == 2) return launch_bwd_stages<D, 2>(m, pre, a, num_sms, stream, launches);
    if (stages == 3) return launch_bwd_stages<D, 3>(m, pre, a, num_sms, stream, launches);
    if (stages == 4) return launch_bwd_stages<D, 4>(m, pre, a, num_sms, stream, launches);
    return cudaErrorInvalidValue;
  } else {
    if (stages == 3) return launch_bwd_stages<D, 3>(m, pre, a, num_sms, stream, launches);
    if (stages == 4) return launch_bwd_stages<D, 4>(m, pre, a, num_sms, stream, launches);
    return cudaErrorInvalidValue;
  }
}

template cudaError_t launch_bwd<64>(const BwdMaps&, const BwdPreArgs&, const BwdArgs&, int, cudaStream_t, int*,
                                    int);
template cudaError_t launch_bwd<128>(const BwdMaps&, const BwdPreArgs&, const BwdArgs&, int, cudaStream_t, int*,
                                     int);

}  // namespace s2
