// S2-Attn backward for sm_100a in one pass over the score tiles: dK, dV and the
// dQ partials from the same P and dS (head dim 128).
//
// The gradient is that of plain softmax attention inside each rolled group
// (LongQLoRA community post, section 03, Shift Short Attention; causal inside
// a group, section 04):
//   dP = dO V^T,  dS = P * (dP - Delta),  dQ = scale dS K,  dK = scale dS^T Q,  dV = P^T dO.
// The split backward (s2_bwd.cu) recomputes S and dP in a second kernel to
// get dQ; here every (kv tile, query sub-tile) pair is visited once and dQ's
// share of it, dQ^T = K^T dS^T (128 x 64, fp32), is added into a caller-owned
// fp32 accumulator [B, H, N, D] by a bulk reduction at L2.  Three kernels run
// in order on one stream: the preprocess (-Delta, -lse log2 e, and zeroes the
// accumulator), this kernel, and s2_bwd_dq_post_kernel (dq = bf16(scale * acc)).
//
// Persistent: one CTA per SM walks its share of 128-row kv tiles (the paired
// schedule of s2_common.cuh); the query side streams in 64-row sub-tiles g,
// for every query head of the kv-head, from the diagonal to the group end.
// Per sub-tile five UMMAs (M = 128, all operands in shared memory):
//   S^T  = K Q^T          -> TMEM (64 columns, one buffer)      issuer A (warp 1)
//   dP^T = V dO^T         -> TMEM (64 columns, one buffer)      issuer B (warp 10)
//   dV  += P^T dO,  P^T from shared memory                      issuer A
//   dK  += dS^T Q,  dS^T from shared memory                     issuer B
//   dQ^T = K^T dS^T       -> TMEM (two 64-column buffers)       issuer C (warp 11)
// Warps 2..9 (thread = kv row = TMEM lane; warps 2..5 query columns 0..31,
// 6..9 columns 32..63) read S^T and dP^T into registers -- which frees their
// TMEM for sub-tile g+1 at once -- and write P^T and dS^T (bf16, 128-byte
// swizzled, K-major for dV/dK and MN-major for dQ^T: the same bytes) into a
// double-buffered shared-memory pair.  When dV, dK and dQ^T of sub-tile g have
// completed, that pair is free again: the same warps copy dQ^T(g) out of TMEM
// into it as fp32 [64 query rows][D] and issuer C sends it to the accumulator
// with one cp.reduce.async.bulk (the 64 query rows of a sub-tile are
// contiguous in the original order: the shift is a whole number of tiles).
// TMEM (512 columns): dV [0, D), dK [D, 2D), S^T [2D, 2D+64), dP^T
// [2D+64, 2D+128), dQ^T [2D+128, 2D+256).  K and V are single-buffered (the
// next item's V is fetched as soon as the last dP^T has read the old one, its
// K once the last S^T and dQ^T have); Q / dO stream through three stages.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "s2_common.cuh"
#include "s2_ptx.cuh"

namespace s2 {

template <int D>
struct FusedCfg {
  static constexpr int STAGES = 3;
  static constexpr int KV_ATOM = kTile * 128;        // one 64-column slab of a 128-row tile
  static constexpr int Q_ATOM = kSub * 128;          // one 64-column slab of a 64-row tile
  static constexpr int KV_BYTES = kTile * D * 2;
  static constexpr int Q_BYTES = kSub * D * 2;
  static constexpr int PS_BYTES = kTile * kSub * 2;  // P^T or dS^T: 128 kv rows x 64 query columns (bf16)
  static constexpr int DQ_BYTES = kSub * D * 4;      // one dQ partial: 64 query rows x D (fp32)
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = KV_BYTES;
  static constexpr int OFF_Q = 2 * KV_BYTES;
  static constexpr int OFF_DO = OFF_Q + STAGES * Q_BYTES;
  static constexpr int OFF_PS = OFF_DO + STAGES * Q_BYTES;  // [2 buffers][P^T, dS^T]
  static constexpr int OFF_ROW = OFF_PS + 4 * PS_BYTES;     // per stage: -lse2[64], -delta[64]
  static constexpr int SMEM_BYTES = OFF_ROW + STAGES * 512 + 1024;  // + alignment slack
  static constexpr uint32_t TM_DV = 0, TM_DK = D, TM_S = 2 * D, TM_DP = 2 * D + 64, TM_DQ = 2 * D + 128;
  static constexpr int THREADS = 384;
  static_assert(D == 128, "dQ^T = K^T dS^T is an M = D UMMA: head dim 128");
  static_assert(DQ_BYTES <= 2 * PS_BYTES, "a dQ partial is staged in one P^T / dS^T buffer pair");
  static_assert(TM_DQ + 2 * kSub <= 512, "TMEM columns");
  static_assert(SMEM_BYTES <= 232448 - 512, "shared memory");
};

__device__ __forceinline__ float4 ldg_nc_f4(const float* p) {
  float4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}

template <int D>
__global__ void __launch_bounds__(384, 1)
    s2_bwd_fused_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmG,
                        const BwdArgs a) {
  using C = FusedCfg<D>;
  constexpr int ST = C::STAGES;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  // bar_mma_done[b]: dV, dK and dQ^T of the last sub-tile on buffer pair b have
  // completed (one commit per issuer); bar_stg_full / bar_buf_free: the dQ
  // partial staged in pair b is written / has been read by the bulk reduction.
  __shared__ __align__(8) uint64_t bar_k, bar_v, bar_k_empty, bar_v_empty, bar_full[ST], bar_empty[ST], bar_s,
      bar_dp, bar_sdp_free, bar_pds[2], bar_mma_done[2], bar_dq_free[2], bar_stg_full[2], bar_buf_free[2],
      bar_acc_full, bar_acc_free, bar_drain[3];
  __shared__ uint32_t tmem_slot;
  __shared__ uint32_t abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Dims& d = a.d;
  const PairSched& ps = a.kv_sched;
  WaitCtx wc{&abort_flag, a.status, a.wait_limit_ns};

  const uint32_t s0 = smem_u32(smem);
  const uint32_t sK = s0 + C::OFF_K, sV = s0 + C::OFF_V;
  auto sQ = [&](int s) { return s0 + C::OFF_Q + s * C::Q_BYTES; };
  auto sG = [&](int s) { return s0 + C::OFF_DO + s * C::Q_BYTES; };
  auto sPS = [&](int b) { return s0 + C::OFF_PS + b * 2 * C::PS_BYTES; };  // P^T; dS^T follows
  auto sRow = [&](int s) { return s0 + C::OFF_ROW + s * 512; };

  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar_k), 1);
    mbar_init(smem_u32(&bar_v), 1);
    mbar_init(smem_u32(&bar_k_empty), 2);  // issuer A after its last S^T, C after its last dQ^T
    mbar_init(smem_u32(&bar_v_empty), 1);  // issuer B after its last dP^T
    for (int s = 0; s < ST; ++s) {
      mbar_init(smem_u32(&bar_full[s]), 1);
      mbar_init(smem_u32(&bar_empty[s]), 2);  // A after dV, B after dK
    }
    mbar_init(smem_u32(&bar_s), 1);
    mbar_init(smem_u32(&bar_dp), 1);
    mbar_init(smem_u32(&bar_sdp_free), 8);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&bar_pds[i]), 8);
      mbar_init(smem_u32(&bar_mma_done[i]), 3);
      mbar_init(smem_u32(&bar_dq_free[i]), 8);
      mbar_init(smem_u32(&bar_stg_full[i]), 8);
      mbar_init(smem_u32(&bar_buf_free[i]), 1);
    }
    mbar_init(smem_u32(&bar_acc_full), 2);
    mbar_init(smem_u32(&bar_acc_free), 8);
    for (int i = 0; i < 3; ++i) mbar_init(smem_u32(&bar_drain[i]), 1);
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
    int gi = 0, nk = 0, nv = 0;
    bool ok = true;
    // Q / dO / row statistics of sub-tile `it` of item w into the next stage
    auto load_stage = [&](const TileWork& w, int sh, int it, int nq) -> bool {
      const int s = gi % ST, f = gi / ST;
      if (f > 0 && !warp_wait(smem_u32(&bar_empty[s]), (f - 1) & 1, wc, 310)) return false;
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
      ++gi;
      return true;
    };
    ItemCursor ic;
    for (ic.first(ps); ok && ic.valid; ic.next(ps)) {
      const TileWork w = kv_item(d, ic.unit, ic.tile);
      const int sh = shift_of_head(d, w.h);
      const int nq = 2 * (d.tiles - w.tile);
      const int iters = d.rep * nq;
      const int tk0 = original_row_kv(d, w.g * d.G + w.tile * kTile, sh);
      // the item's first stages need only free stages, not the new K / V
      const int pre = iters < ST ? iters : ST;
      for (int it = 0; ok && it < pre; ++it) ok = load_stage(w, sh, it, nq);
      if (!ok) break;
      if (nv > 0 && !warp_wait(smem_u32(&bar_v_empty), (nv - 1) & 1, wc, 311)) break;
      if (elect_one()) {
        mbar_arrive_expect_tx(smem_u32(&bar_v), C::KV_BYTES);
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(sV + c * C::KV_ATOM, &tmV, smem_u32(&bar_v), c * 64, w.kvh, tk0, w.b);
      }
      __syncwarp();
      ++nv;
      if (nk > 0 && !warp_wait(smem_u32(&bar_k_empty), (nk - 1) & 1, wc, 312)) break;
      if (elect_one()) {
        mbar_arrive_expect_tx(smem_u32(&bar_k), C::KV_BYTES);
        for (int c = 0; c < D / 64; ++c)
          tma_load_4d(sK + c * C::KV_ATOM, &tmK, smem_u32(&bar_k), c * 64, w.kvh, tk0, w.b);
      }
      __syncwarp();
      ++nk;
      for (int it = pre; ok && it < iters; ++it) ok = load_stage(w, sh, it, nq);
    }
    if (*wc.abort && lane == 0) {
      // never leave copies in flight into shared memory: wait (bounded) for
      // the last fill of K, V and every stage
      if (nk > 0) drain_wait(smem_u32(&bar_k), (nk - 1) & 1);
      if (nv > 0) drain_wait(smem_u32(&bar_v), (nv - 1) & 1);
      for (int s = 0; s < ST && s < gi; ++s) drain_wait(smem_u32(&bar_full[s]), ((gi - 1 - s) / ST) & 1);
    }
  } else if (warp == 1 || warp == 10) {
    // ------------------------------------------------------------ issuers A and B
    // A (warp 1): S^T = K Q^T and dV += P^T dO.  B (warp 10): dP^T = V dO^T
    // and dK += dS^T Q.  Each issues the next sub-tile's score UMMAs before
    // this sub-tile's gradient UMMAs (the scores' TMEM is free as soon as the
    // elementwise warps have read it), except at the end of an item, where the
    // gradient UMMAs go first so the accumulators are ready for the epilogue
    // while the next item's K / V arrive.
    const bool A = (warp == 1);
    const uint32_t idS = make_idesc_bf16(128, kSub, 0, 0);  // S^T, dP^T: both operands K-major
    const uint32_t idG = make_idesc_bf16(128, D, 0, 1);     // dV, dK: A K-major, B MN-major
    const uint64_t dX0 = make_sdesc_sw128(A ? sK : sV, 16, 1024);                // K-major A of S^T / dP^T
    const uint64_t dYk = make_sdesc_sw128(A ? sQ(0) : sG(0), 16, 1024);          // K-major B of S^T / dP^T
    const uint64_t dZm = make_sdesc_sw128(A ? sG(0) : sQ(0), C::Q_ATOM, 1024);   // MN-major B of dV / dK
    const uint64_t dP0 = make_sdesc_sw128(sPS(0) + (A ? 0 : C::PS_BYTES), 16, 1024);  // K-major A: P^T / dS^T
    const uint32_t tm_sp = tmem + (A ? C::TM_S : C::TM_DP);
    const uint32_t tm_acc = tmem + (A ? C::TM_DV : C::TM_DK);
    const uint32_t bar_sp = smem_u32(A ? &bar_s : &bar_dp);
    const uint32_t bar_kv = smem_u32(A ? &bar_k : &bar_v);
    const uint32_t bar_kv_empty = smem_u32(A ? &bar_k_empty : &bar_v_empty);
    auto issue_sp = [&](const DkvCursor& c, int g) -> bool {
      if (c.it == 0 && !warp_wait(bar_kv, c.ic.n & 1, wc, A ? 320 : 330)) return false;
      if (!warp_wait(smem_u32(&bar_full[g % ST]), (g / ST) & 1, wc, A ? 321 : 331)) return false;
      if (g > 0 && !warp_wait(smem_u32(&bar_sdp_free), (g - 1) & 1, wc, A ? 322 : 332)) return false;
      tc_fence_after();
      const uint64_t dy = sdesc_advance(dYk, (g % ST) * C::Q_BYTES);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ko = (kk >> 2) * C::KV_ATOM + (kk & 3) * 32;
          const uint32_t qo = (kk >> 2) * C::Q_ATOM + (kk & 3) * 32;
          umma_ss(tm_sp, sdesc_advance(dX0, ko), sdesc_advance(dy, qo), idS, kk > 0);
        }
        umma_commit(bar_sp);
        if (c.it == c.iters - 1) umma_commit(bar_kv_empty);  // the item's last reader of K (A) / V (B)
      }
      __syncwarp();
      return true;
    };
    auto issue_grad = [&](const DkvCursor& c, int g) -> bool {
      if (!warp_wait(smem_u32(&bar_pds[g & 1]), (g >> 1) & 1, wc, A ? 323 : 333)) return false;
      if (c.it == 0 && c.ic.n > 0 && !warp_wait(smem_u32(&bar_acc_free), (c.ic.n - 1) & 1, wc, A ? 324 : 334))
        return false;
      tc_fence_after();
      const int s = g % ST;
      const uint64_t da = sdesc_advance(dP0, (g & 1) * 2 * C::PS_BYTES);
      const uint64_t dz = sdesc_advance(dZm, s * C::Q_BYTES);
      const bool last = (c.it == c.iters - 1);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < kSub / 16; ++kk)
          umma_ss(tm_acc, sdesc_advance(da, kk * 32), sdesc_advance(dz, kk * 2048), idG, (c.it > 0 || kk > 0));
        umma_commit(smem_u32(&bar_empty[s]));
        umma_commit(smem_u32(&bar_mma_done[g & 1]));
        if (last) umma_commit(smem_u32(&bar_acc_full));
      }
      __syncwarp();
      return true;
    };
    DkvCursor cur;
    cur.first(d, ps);
    bool ok = true;
    if (cur.ic.valid) ok = issue_sp(cur, 0);
    for (int g = 0; ok && cur.ic.valid; ++g) {
      DkvCursor nx = cur;
      nx.next(d, ps);
      const bool boundary = (cur.it == cur.iters - 1);
      if (!boundary && nx.ic.valid && !(ok = issue_sp(nx, g + 1))) break;
      if (!(ok = issue_grad(cur, g))) break;
      if (boundary && nx.ic.valid && !(ok = issue_sp(nx, g + 1))) break;
      cur = nx;
    }
    if (elect_one()) {
      umma_commit(smem_u32(&bar_drain[A ? 0 : 1]));
      drain_wait(smem_u32(&bar_drain[A ? 0 : 1]), 0);
    }
    __syncwarp();
  } else if (warp == 11) {
    // ------------------------------------------------------------ issuer C
    // dQ^T(g) = K^T dS^T(g) into TMEM buffer g & 1, then the bulk reduction of
    // the previous sub-tile's partial once the elementwise warps staged it.
    const uint32_t idQ = make_idesc_bf16(128, kSub, 1, 1);            // A = K^T (MN-major), B = dS^T (MN-major)
    const uint64_t dKm = make_sdesc_sw128(sK, C::KV_ATOM, 1024);        // M = D over the two 64-column slabs
    const uint64_t dSm = make_sdesc_sw128(sPS(0) + C::PS_BYTES, C::PS_BYTES, 1024);  // N = 64: one slab
    auto issue_dq = [&](const DkvCursor& c, int g) -> bool {
      if (!warp_wait(smem_u32(&bar_pds[g & 1]), (g >> 1) & 1, wc, 340)) return false;
      if (g >= 2 && !warp_wait(smem_u32(&bar_dq_free[g & 1]), ((g - 2) >> 1) & 1, wc, 341)) return false;
      tc_fence_after();
      const uint64_t db = sdesc_advance(dSm, (g & 1) * 2 * C::PS_BYTES);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          umma_ss(tmem + C::TM_DQ + (g & 1) * kSub, sdesc_advance(dKm, kk * 2048), sdesc_advance(db, kk * 2048), idQ,
                  kk > 0);
        umma_commit(smem_u32(&bar_mma_done[g & 1]));
        if (c.it == c.iters - 1) umma_commit(smem_u32(&bar_k_empty));  // the item's last reader of K
      }
      __syncwarp();
      return true;
    };
    auto reduce = [&](const DkvCursor& c, int g) -> bool {
      if (!warp_wait(smem_u32(&bar_stg_full[g & 1]), (g >> 1) & 1, wc, 342)) return false;
      const TileWork& w = c.w;
      const int h = w.kvh * d.rep + c.it / c.nq;
      const int i64 = 2 * w.tile + c.it % c.nq;
      const int tq0 = original_row(d, w.g * d.G + i64 * kSub, shift_of_head(d, w.h));
      float* dst = a.dqacc + ((static_cast<size_t>(w.b) * d.H + h) * d.N + tq0) * D;
      if (elect_one()) {
        bulk_reduce_add_f32(dst, sPS(g & 1), C::DQ_BYTES);
        bulk_commit_group();
        bulk_wait_read_all();  // the staging pair may be overwritten from here on
        mbar_arrive(smem_u32(&bar_buf_free[g & 1]));
      }
      __syncwarp();
      return true;
    };
    DkvCursor cur, prev;
    cur.first(d, ps);
    bool ok = true;
    int g = 0;
    for (; ok && cur.ic.valid; ++g) {
      if (!(ok = issue_dq(cur, g))) break;
      if (g >= 1 && !(ok = reduce(prev, g - 1))) break;
      prev = cur;
      cur.next(d, ps);
    }
    if (ok && g >= 1) reduce(prev, g - 1);
    if (elect_one()) {
      bulk_wait_all();  // every reduction performed before the CTA ends
      umma_commit(smem_u32(&bar_drain[2]));
      drain_wait(smem_u32(&bar_drain[2]), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ P^T, dS^T, dQ staging, epilogue
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = quarter * 32 + lane;  // kv row of the tile (TMEM lane); in dQ^T the head-dim index
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float sl2 = a.scale_log2;
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    const uint32_t sw = static_cast<uint32_t>(row & 7);
    bool ok = true;
    // dQ^T of sub-tile gp out of TMEM into its buffer pair as fp32 [64][D]
    auto stage_dq = [&](int gp) -> bool {
      const int b = gp & 1;
      if (!warp_wait(smem_u32(&bar_mma_done[b]), (gp >> 1) & 1, wc, 353)) return false;
      tc_fence_after();
      uint32_t r[32];
      tmem_ld32(tmem + lane_off + C::TM_DQ + b * kSub + half * 32, r);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar_dq_free[b]));
      const uint32_t stg = sPS(b) + (half * 32 * D + row) * 4;
#pragma unroll
      for (int j = 0; j < 32; ++j) st_shared_f32(stg + j * D * 4, __uint_as_float(r[j]));
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar_stg_full[b]));
      return true;
    };
    DkvCursor cur;
    cur.first(d, ps);
    int g = 0;
    for (; cur.ic.valid; ++g) {
      const int s = g % ST, b = g & 1;
      const int qoff = (cur.it % cur.nq) * kSub;  // query sub-tile start minus kv tile start (rolled)
      ok = warp_wait(smem_u32(&bar_full[s]), (g / ST) & 1, wc, 350) &&
           warp_wait(smem_u32(&bar_s), g & 1, wc, 351) && warp_wait(smem_u32(&bar_dp), g & 1, wc, 352);
      if (!ok) break;
      tc_fence_after();
      // row statistics of this half's 32 query rows: -lse*log2e at +0, -Delta at +256 bytes
      const uint32_t l4 = sRow(s) + half * 128, d4 = l4 + 256;
      float4 lv[8], dv4[8];
#pragma unroll
      for (int c4 = 0; c4 < 8; ++c4) {
        lv[c4] = lds_f4(l4 + c4 * 16);
        dv4[c4] = lds_f4(d4 + c4 * 16);
      }
      uint32_t sr[32], dr[32];
      tmem_ld32(tmem + lane_off + C::TM_S + half * 32, sr);
      tmem_ld32(tmem + lane_off + C::TM_DP + half * 32, dr);
      tmem_wait_ld();
      // S^T / dP^T are in registers: the next sub-tile's scores may overwrite them
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar_sdp_free));
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
      // the pair held the dQ partial of sub-tile g-2: wait until the bulk
      // reduction has read it
      if (g >= 2) {
        ok = warp_wait(smem_u32(&bar_buf_free[b]), ((g - 2) >> 1) & 1, wc, 354);
        if (!ok) break;
      }
      // P^T and dS^T rows (bf16, 128-byte swizzled): this thread's 32 query
      // columns are 16-byte chunks 4*half .. 4*half+3 of its row
      const uint32_t prow = sPS(b) + row * 128;
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        const uint32_t off = ((static_cast<uint32_t>(half * 4 + c4) ^ sw) << 4);
        st_shared_v4(prow + off, pk[4 * c4], pk[4 * c4 + 1], pk[4 * c4 + 2], pk[4 * c4 + 3]);
        st_shared_v4(prow + C::PS_BYTES + off, dk[4 * c4], dk[4 * c4 + 1], dk[4 * c4 + 2], dk[4 * c4 + 3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar_pds[b]));
      if (g >= 1 && !(ok = stage_dq(g - 1))) break;
      if (cur.it == cur.iters - 1) {
        // ---------------------------------------------------- dK / dV epilogue of this item
        ok = warp_wait(smem_u32(&bar_acc_full), cur.ic.n & 1, wc, 355);
        if (!ok) break;
        tc_fence_after();
        const TileWork& w = cur.w;
        const int tk0 = original_row(d, w.g * d.G + w.tile * kTile, shift_of_head(d, w.h));
        const size_t grow = (static_cast<size_t>(w.b) * d.N + tk0 + row) * d.Hkv + w.kvh;
        // this thread's columns: [32 half, 32 half + 32) and the same + D/2, so
        // that rotary pairs (i, i + D/2) stay in one thread
        __nv_bfloat16* dvrow = static_cast<__nv_bfloat16*>(a.dv) + grow * D + half * 32;
        __nv_bfloat16* dkrow = static_cast<__nv_bfloat16*>(a.dk) + grow * D + half * 32;
        uint32_t r[2][32], r2[2][32];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          tmem_ld32(tmem + lane_off + C::TM_DV + c * (D / 2) + half * 32, r[c]);
          tmem_ld32(tmem + lane_off + C::TM_DK + c * (D / 2) + half * 32, r2[c]);
        }
        tmem_wait_ld();
        // dV / dK are out of TMEM: the next item's first gradient UMMAs may start
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bar_acc_free));
        if (a.rope != nullptr) {
          // the inputs were rotated at token tk0 + row: turn dK back by -angle
          const float4* tp = reinterpret_cast<const float4*>(a.rope + (static_cast<size_t>(tk0 + row) * (D / 2) +
                                                                      half * 32) * 2);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float4 cs = tp[j];  // (cos, sin) of pairs 2j, 2j+1 of this thread's 32
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const float co = u ? cs.z : cs.x, si = u ? cs.w : cs.y;
              const float x1 = __uint_as_float(r2[0][2 * j + u]), x2 = __uint_as_float(r2[1][2 * j + u]);
              r2[0][2 * j + u] = __float_as_uint(fmaf(x1, co, x2 * si));
              r2[1][2 * j + u] = __float_as_uint(fmaf(x2, co, -x1 * si));
            }
          }
        }
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          if (a.kv_v8) {
            store_row32_v8(dvrow + c * (D / 2), r[c], 1.f);
            store_row32_v8(dkrow + c * (D / 2), r2[c], a.scale);
          } else {
            store_row32(dvrow + c * (D / 2), r[c], 1.f);
            store_row32(dkrow + c * (D / 2), r2[c], a.scale);
          }
        }
      }
      cur.next(d, ps);
    }
    if (ok && g >= 1) stage_dq(g - 1);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// dq = bf16(scale * acc), turned back by the rotary table when the inputs
// were rotated: one block per 128 rows of one (batch, head); each thread takes
// 8 rotary pairs (i, i + D/2) of a row, so the back-rotation stays in-thread.
template <int D>
__global__ void __launch_bounds__(256) s2_bwd_dq_post_kernel(const float* dqacc, __nv_bfloat16* dq, const Dims d,
                                                             float scale, const float* rope) {
  constexpr int TPR = D / 16;        // threads per row, 8 pairs each
  constexpr int RPP = 256 / TPR;     // rows per pass
  constexpr int PASSES = kTile / RPP;
  const int tid = threadIdx.x, c = tid % TPR, rs = tid / TPR;
  const int tblk = d.N / kTile;
  const long long tasks = static_cast<long long>(d.B) * d.H * tblk;
  for (long long task = blockIdx.x; task < tasks; task += gridDim.x) {
    const long long bh = task / tblk;
    const int t0 = static_cast<int>(task - bh * tblk) * kTile;
    const int h = static_cast<int>(bh % d.H), b = static_cast<int>(bh / d.H);
#pragma unroll 2
    for (int p = 0; p < PASSES; ++p) {
      const int t = t0 + p * RPP + rs;
      const float* src = dqacc + (static_cast<size_t>(bh) * d.N + t) * D + c * 8;
      float x1[8], x2[8];
      const float4 a0 = ldg_nc_f4(src), a1 = ldg_nc_f4(src + 4);
      const float4 b0 = ldg_nc_f4(src + D / 2), b1 = ldg_nc_f4(src + D / 2 + 4);
      x1[0] = a0.x; x1[1] = a0.y; x1[2] = a0.z; x1[3] = a0.w; x1[4] = a1.x; x1[5] = a1.y; x1[6] = a1.z; x1[7] = a1.w;
      x2[0] = b0.x; x2[1] = b0.y; x2[2] = b0.z; x2[3] = b0.w; x2[4] = b1.x; x2[5] = b1.y; x2[6] = b1.z; x2[7] = b1.w;
      if (rope != nullptr) {
        const float4* tp = reinterpret_cast<const float4*>(rope + (static_cast<size_t>(t) * (D / 2) + c * 8) * 2);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float4 cs = tp[j];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int k = 2 * j + u;
            const float co = u ? cs.z : cs.x, si = u ? cs.w : cs.y;
            const float y1 = fmaf(x1[k], co, x2[k] * si), y2 = fmaf(x2[k], co, -x1[k] * si);
            x1[k] = y1;
            x2[k] = y2;
          }
        }
      }
      __nv_bfloat16* dst = dq + ((static_cast<size_t>(b) * d.N + t) * d.H + h) * D + c * 8;
      *reinterpret_cast<uint4*>(dst) =
          make_uint4(pack_bf16x2(x1[0] * scale, x1[1] * scale), pack_bf16x2(x1[2] * scale, x1[3] * scale),
                     pack_bf16x2(x1[4] * scale, x1[5] * scale), pack_bf16x2(x1[6] * scale, x1[7] * scale));
      *reinterpret_cast<uint4*>(dst + D / 2) =
          make_uint4(pack_bf16x2(x2[0] * scale, x2[1] * scale), pack_bf16x2(x2[2] * scale, x2[3] * scale),
                     pack_bf16x2(x2[4] * scale, x2[5] * scale), pack_bf16x2(x2[6] * scale, x2[7] * scale));
    }
  }
}

template <int D>
cudaError_t launch_bwd_fused(const BwdMaps& m, const BwdPreArgs& pre, const BwdArgs& a, int num_sms,
                             cudaStream_t stream, int* launches) {
  using C = FusedCfg<D>;
  if (cudaFuncSetAttribute(s2_bwd_fused_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
      cudaSuccess)
    return cudaErrorInvalidValue;
  cudaError_t e = launch_bwd_pre<D>(pre, num_sms, stream);
  if (e != cudaSuccess) return e;
  const int grid = pair_grid(a.kv_sched, num_sms);
  prof_before(stream, kKernelBwdFused);
  s2_bwd_fused_kernel<D><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(m.q64, m.k128, m.v128, m.g64, a);
  e = cudaGetLastError();
  prof_after(stream);
  if (e != cudaSuccess) return e;
  const long long tasks = static_cast<long long>(a.d.B) * a.d.H * (a.d.N / kTile);
  const int post_grid = static_cast<int>(tasks < 8LL * num_sms ? tasks : 8LL * num_sms);
  prof_before(stream, kKernelBwdDqPost);
  s2_bwd_dq_post_kernel<D><<<post_grid, 256, 0, stream>>>(a.dqacc, static_cast<__nv_bfloat16*>(a.dq), a.d, a.scale,
                                                           a.rope);
  e = cudaGetLastError();
  prof_after(stream);
  if (launches) *launches = 3;
  return e;
}

template cudaError_t launch_bwd_fused<128>(const BwdMaps&, const BwdPreArgs&, const BwdArgs&, int, cudaStream_t,
                                           int*);

}  // namespace s2
