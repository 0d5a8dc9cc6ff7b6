// Thin inline-PTX layer for sm_100a: mbarriers with bounded waits, TMA tile
// loads, tcgen05 (TMEM allocation, UMMA issue/commit, TMEM load/store) and the
// shared-memory matrix descriptors the UMMA reads its operands through.
//
// Every wait here is bounded by wall-clock time (the %globaltimer register):
// a wait that runs out records an error word in global memory, raises a CTA-
// local abort flag and returns false, so a kernel never spins forever.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

namespace s2 {

// ----------------------------------------------------------------- status

// Device status word layout (the first 16 bytes of the caller's workspace,
// or a kernel's own status pointer): [0] error code, [1] where it happened.
enum DeviceError : uint32_t {
  kDevOk = 0,
  kDevWaitTimeout = 5,  // matches S2ATTN_ERR_DEVICE_TIMEOUT in the C ABI
};

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// One lane of a converged warp is elected (elect.sync).  Issuing UMMAs and
// TMA copies from an elected lane of a converged warp, instead of from a
// lane-0 branch, keeps the issuing warp fast when the other warps on its SM
// sub-partition are issuing heavily (measured: about 3.4x fewer cycles per
// UMMA batch under full contention).
__device__ __forceinline__ bool elect_one() {
  uint32_t e;
  asm volatile(
      "{\n\t.reg .pred P1;\n\t"
      "elect.sync _|P1, 0xffffffff;\n\t"
      "selp.b32 %0, 1, 0, P1;\n\t}"
      : "=r"(e));
  return e != 0;
}

// ----------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  // make mbarrier.init visible to the async proxy (TMA, tcgen05.commit)
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Shared state every bounded wait consults.  `abort` lives in shared memory:
// once any thread of the CTA gives up, every other wait returns at once.
struct WaitCtx {
  volatile uint32_t* abort;  // CTA-local flag (shared memory)
  uint32_t* status;          // global status word pair, may be null
  uint64_t limit_ns;         // per-wait time limit
};

static __device__ __noinline__ void record_timeout(const WaitCtx& w, uint32_t where) {
  *w.abort = 1u;
  if (w.status != nullptr) {
    if (atomicCAS(w.status, 0u, (uint32_t)kDevWaitTimeout) == 0u) w.status[1] = where;
  }
}

// Wait for phase `parity` of mbarrier `bar` to complete.  Returns false (after
// recording the failure) if the limit runs out or another thread aborted.
// A parity names phase k only while the barrier's open phase is k or k+1:
// with k+2 open (k and k+1 complete) the open phase has k's parity and the
// wait blocks; with k-1 open the open phase's parity differs from k's and the
// wait passes at once.  Every caller keeps its barrier within that window:
// phase k+1 needs something the waiter does after the wait, and phase k-1 is
// complete before it (by its own earlier wait, or by a wait that implies it).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, const WaitCtx& w,
                                          uint32_t where) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0u) {
      if (*w.abort) return false;
      if (globaltimer_ns() - t0 > w.limit_ns) {
        record_timeout(w, where);
        return false;
      }
    }
  }
}

// Bounded wait by a whole converged warp; every lane gets the same answer.
// Every lane polls (one warp instruction per poll): measured faster than
// lane 0 polling and broadcasting its answer, both for the single-thread
// producer / issuer warps and for the compute warps.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const WaitCtx& w,
                                          uint32_t where) {
  const bool ok = mbar_wait(bar, parity, w, where);
  return __all_sync(0xffffffffu, ok);
}

// Bounded wait used only on the way out of an aborted kernel, to let copies
// and UMMAs already in flight land before shared memory / TMEM are released.
// Ignores the abort flag; gives up silently after ~50 ms.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > 50000000ull) return;
  }
}

__device__ __forceinline__ float neg_inf() { return __int_as_float(0xff800000); }

// ----------------------------------------------------------------- TMA

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 4-D tiled load (coordinates innermost first) completing on mbarrier `bar`.
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
      : "memory");
}

// 2-D tiled load (coordinates innermost first) completing on mbarrier `bar`.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

// 2-D tiled TMA store shared -> global through the issuing thread's bulk group
// (no coordinate may be negative; rows or columns past the tensor are clipped).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int c0, int c1) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(c0), "r"(c1)
               : "memory");
}

// Tiled TMA store shared -> global, completed through the issuing thread's
// bulk group.  The innermost coordinate times the element size must be a
// multiple of 16 bytes and no coordinate may be negative.
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, uint32_t src, int c0, int c1, int c2,
                                             int c3) {
  asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
               : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until every committed bulk store of this thread has read its shared-
// memory source (the source may then be reused; the global writes may still
// be in flight).
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// Wait until every committed bulk operation of this thread has completed
// (its global writes or reductions are performed).
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Untiled bulk reduction shared -> global: dst[i] += src[i] for `bytes` / 4
// fp32 values, performed at L2; both addresses 16-byte aligned, bytes % 16 == 0.
// Completes through the issuing thread's bulk group.
__device__ __forceinline__ void bulk_reduce_add_f32(void* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(
                   reinterpret_cast<uint64_t>(dst)),
               "r"(src), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void st_shared_u16(uint32_t addr, uint16_t v) {
  asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}

__device__ __forceinline__ void st_shared_f32(uint32_t addr, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

// Plain (untiled) bulk copy global -> shared, 16-byte aligned, size % 16 == 0.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// Order this thread's generic-proxy shared-memory writes before later
// async-proxy reads (UMMA operands, TMA stores).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ----------------------------------------------------------------- tcgen05

// TMEM allocation: executed by one whole warp; the base address is written to
// shared memory at `dst`.
__device__ __forceinline__ void tmem_alloc(uint32_t dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]   (kind::f16, one CTA)
__device__ __forceinline__ void umma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]   (kind::f16, one CTA)
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when every UMMA this thread issued so far has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread t of the warp receives
// lane (base lane + t), columns [col, col + 32).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns (as tmem_ld32, half as wide).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

// ----------------------------------------------------------------- descriptors

// Instruction descriptor, kind::f16: bf16 A and B, fp32 accumulator, M x N,
// A/B major-ness (0 = K-major, 1 = MN-major).
__host__ __device__ constexpr uint32_t make_idesc_bf16(int M, int N, int a_mn_major,
                                                       int b_mn_major) {
  return (1u << 4)                                 // accumulator format: f32
         | (1u << 7)                               // A format: bf16
         | (1u << 10)                              // B format: bf16
         | ((uint32_t)a_mn_major << 15)            // A major
         | ((uint32_t)b_mn_major << 16)            // B major
         | ((uint32_t)(N >> 3) << 17)              // N / 8
         | ((uint32_t)(M >> 4) << 24);             // M / 16
}

// Shared-memory matrix descriptor for a 128-byte-swizzled operand.
//   start: shared address (bytes), lbo / sbo: leading / stride byte offsets.
// Field layout: start>>4 in [0,14), lbo>>4 in [16,30), sbo>>4 in [32,46),
// descriptor version 1 in [46,48), layout type SWIZZLE_128B (2) in [61,64).
__device__ __forceinline__ uint64_t make_sdesc_sw128(uint32_t start, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((start >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}

// The same for a 64-byte-swizzled operand (layout type SWIZZLE_64B, 4): rows
// of 64 bytes, the swizzle pattern repeating every 8 rows (512 bytes).
__device__ __forceinline__ uint64_t make_sdesc_sw64(uint32_t start, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((start >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)4u << 61;
  return d;
}

// The descriptor of the same operand `bytes` further on in shared memory.
// The start-address field holds address >> 4 in the low 14 bits and shared
// addresses stay below 256 KiB, so the add never carries out of the field.
// With `bytes` a compile-time constant this is a single integer add, which
// keeps the single-thread UMMA issue loop short (a descriptor rebuilt per
// instruction costs a long dependent chain per UMMA).
__device__ __forceinline__ uint64_t sdesc_advance(uint64_t desc, uint32_t bytes) {
  return desc + static_cast<uint64_t>(bytes >> 4);
}

// ----------------------------------------------------------------- math

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// max(a, b, c) in one instruction (sm_100 three-input max; NaN inputs are
// ignored as in fmaxf).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Two floats -> packed bf16x2 (round to nearest even); lo in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Packed pairs of fp32 (sm_100 f32x2 arithmetic): one instruction for two
// lanes of work, which halves the issue slots the elementwise warps take.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t v;
  asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "f"(lo), "f"(hi));
  return v;
}
__device__ __forceinline__ float f2_lo(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float f2_hi(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// bf16x2 (round to nearest even) of a packed fp32 pair
__device__ __forceinline__ uint32_t f2_to_bf16x2(uint64_t v) { return pack_bf16x2(f2_lo(v), f2_hi(v)); }

// P for 64 scores of one query row: p = 2^(s * sl2 - m), packed to bf16
// pairs in pk; returns the fp32 sum.  Arguments and sums use packed f32x2
// arithmetic, the exponentials the MUFU (ex2.approx).
__device__ __forceinline__ float softmax_row64(const uint32_t (&s0)[32], const uint32_t (&s1)[32], float sl2,
                                               float m, uint32_t (&pk)[32]) {
  const uint64_t sc2 = f2_pack(sl2, sl2), nm2 = f2_pack(-m, -m);
  uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    const uint32_t* src = (c < 16) ? s0 : s1;
    const uint64_t x = f2_fma(f2_pack(__uint_as_float(src[(2 * c) & 31]), __uint_as_float(src[(2 * c + 1) & 31])),
                              sc2, nm2);
    const uint64_t p = f2_pack(ex2_approx(f2_lo(x)), ex2_approx(f2_hi(x)));
    pk[c] = f2_to_bf16x2(p);
    acc[c & 3] = f2_add(acc[c & 3], p);
  }
  const uint64_t s = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
  return f2_lo(s) + f2_hi(s);
}

// The same for 32 keys (one 32-column TMEM load): 16 packed pairs.  The
// forward writes P in 16-column pieces so that no more than 16 packed values
// are live beside the 128 scores of a row.
__device__ __forceinline__ float softmax_row32(const uint32_t (&s0)[32], float sl2, float m, uint32_t (&pk)[16]) {
  const uint64_t sc2 = f2_pack(sl2, sl2), nm2 = f2_pack(-m, -m);
  uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const uint64_t x = f2_fma(f2_pack(__uint_as_float(s0[2 * c]), __uint_as_float(s0[2 * c + 1])), sc2, nm2);
    const uint64_t p = f2_pack(ex2_approx(f2_lo(x)), ex2_approx(f2_hi(x)));
    pk[c] = f2_to_bf16x2(p);
    acc[c & 3] = f2_add(acc[c & 3], p);
  }
  const uint64_t s = f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3]));
  return f2_lo(s) + f2_hi(s);
}

// Explicit shared-memory vector load (a pointer into dynamic shared memory
// that went through integer alignment arithmetic is generic to the compiler,
// and generic loads take the long-latency path).
__device__ __forceinline__ float4 lds_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ uint4 lds_u4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// Table lookup across the warp: every lane holds one entry, lane l the entry
// l mod 16 (so lanes 16..31 repeat 0..15), and each lane reads the lane named
// by bits [4:0] of `idx` (shfl.sync idx mode with clamp 31 and no segment
// mask uses exactly those bits).  A 4-bit code in the low bits of idx selects
// its entry whatever bit 4 holds, so callers need not mask idx.  All 32 lanes
// must take part.
__device__ __forceinline__ float warp_lut16(float table, uint32_t idx) {
  float r;
  asm volatile("shfl.sync.idx.b32 %0, %1, %2, 0x1f, 0xffffffff;" : "=f"(r) : "f"(table), "r"(idx));
  return r;
}

// One 32-byte global store (a whole DRAM sector); the address must be 32-byte
// aligned.
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t (&v)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(v[0]), "r"(v[1]),
               "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// ----------------------------------------------------------------- row stores

// 32 fp32 values (bit patterns) times `scale` -> 32 bf16 at dst (64 bytes, 16-byte aligned).
__device__ __forceinline__ void store_row32(__nv_bfloat16* dst, const uint32_t (&r)[32], float scale) {
  uint4* out = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q)
    out[q] = make_uint4(pack_bf16x2(__uint_as_float(r[8 * q]) * scale, __uint_as_float(r[8 * q + 1]) * scale),
                        pack_bf16x2(__uint_as_float(r[8 * q + 2]) * scale, __uint_as_float(r[8 * q + 3]) * scale),
                        pack_bf16x2(__uint_as_float(r[8 * q + 4]) * scale, __uint_as_float(r[8 * q + 5]) * scale),
                        pack_bf16x2(__uint_as_float(r[8 * q + 6]) * scale, __uint_as_float(r[8 * q + 7]) * scale));
}

// The same as two 32-byte stores (whole DRAM sectors); dst 32-byte aligned.
__device__ __forceinline__ void store_row32_v8(__nv_bfloat16* dst, const uint32_t (&r)[32], float scale) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t v[8];
#pragma unroll
    for (int q = 0; q < 8; ++q)
      v[q] = pack_bf16x2(__uint_as_float(r[16 * h + 2 * q]) * scale, __uint_as_float(r[16 * h + 2 * q + 1]) * scale);
    st_global_v8(dst + 16 * h, v);
  }
}

}  // namespace s2
