/*
 * s2attn.h - C ABI of the B200 (sm_100a) shifted sparse attention library.
 *
 * Operation (S2-Attn, "shift short attention").  LongQLoRA community post,
 * section 03 (Method, Background: Shift Short Attention) and LongLoRA abstract
 * ("LongLoRA: Efficient Fine-tuning of Long-Context Large Language Models"):
 * the length-N sequence is cut into groups of G rows, softmax attention runs
 * only inside each group, and attention between groups is recovered by
 * shifting half of the heads.  Concretely, for query head h:
 *
 *   shift s_h = G/2 when G < N and h >= H/2 (integer division), else 0;
 *   rolled row r holds original row t = (r + s_h) mod N (wrap-around);
 *   group of rolled row r is r / G; attention is causal in rolled order;
 *   kv-head of query head h is h / (H / Hkv) (grouped-query attention);
 *   scale = 1/sqrt(D); results are stored back at original rows.
 *
 * G == N is plain dense causal attention (no shift), the comparison path
 * (LongQLoRA post, sections 03-04: global attention at inference).
 *
 * Layout (all row-major, innermost dimension last):
 *   q, o, dO, dq : bf16 [B, N, H, D]
 *   k, v, dk, dv : bf16 [B, N, Hkv, D]
 *   lse          : fp32 [B, H, N], natural-log log-sum-exp of each query row
 *                  (scaled scores), indexed by original position.
 * All pointers are DEVICE pointers and must be 16-byte aligned.
 *
 * Ownership: the caller allocates and owns every buffer it passes, including
 * the backward workspace; the library never allocates or frees device memory
 * at run time.  Its own device state is fixed at module load: the forward's
 * status block and the scratch array of s2attn_bwd_noalloc (below), both
 * file-scope __device__ arrays held by every GPU that loads the library.
 * Calls are asynchronous on `stream` (0 = legacy default stream) and perform
 * no host synchronisation, except s2attn_device_status.
 *
 * Errors: arguments are validated before anything is launched; a non-zero
 * return means nothing was launched (except S2ATTN_ERR_CUDA, which reports a
 * launch failure).  No C++ exception crosses this boundary.  A kernel that
 * gives up a bounded wait records S2ATTN_ERR_DEVICE_TIMEOUT in its device
 * status word, read back with s2attn_device_status.
 */
#ifndef S2ATTN_H_
#define S2ATTN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define S2ATTN_API __attribute__((visibility("default")))
#else
#define S2ATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  S2ATTN_OK = 0,
  S2ATTN_ERR_INVALID_ARG = 1,    /* null pointer, non-positive size, N % G, H % Hkv, ... */
  S2ATTN_ERR_UNSUPPORTED = 2,    /* shape outside what the kernels implement (see below) */
  S2ATTN_ERR_MISALIGNED = 3,     /* a pointer is not 16-byte aligned */
  S2ATTN_ERR_CUDA = 4,           /* a CUDA runtime/driver call or a launch failed */
  S2ATTN_ERR_DEVICE_TIMEOUT = 5, /* a kernel's bounded wait ran out (device status word) */
  S2ATTN_ERR_WORKSPACE = 6       /* workspace missing or smaller than required */
} s2attn_status;

/* Opaque CUDA stream handle (cudaStream_t) without pulling in CUDA headers. */
typedef void* s2attn_stream_t;

/*
 * Shapes.  G <= N, N % G == 0 and H % Hkv == 0 belong to the definition
 * (S2ATTN_ERR_INVALID_ARG otherwise).  Supported (S2ATTN_ERR_UNSUPPORTED otherwise):
 *   D in {64, 128};  N % 128 == 0;  G % 128 == 0;
 *   when G < N (shifted heads exist): G % 256 == 0, so the G/2 shift is a
 *   whole number of 128-row tiles, and (H/2) % (H/Hkv) == 0, so the query
 *   heads of one kv-head share one shift;  a device of compute capability 10.0.
 */

/*
 * Forward.  o = S2Attn(q, k, v) and lse, as defined above.
 *   q, k, v: inputs; o, lse: outputs (fully overwritten).
 *   B, H, Hkv, N, D, G: batch, query heads, kv heads, sequence length,
 *   head dim, group size (G == N: dense causal).
 */
S2ATTN_API int s2attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
               int B, int H, int Hkv, int N, int D, int G, s2attn_stream_t stream);

/*
 * Bytes of device workspace s2attn_bwd needs: a 256-byte device status block,
 * then two fp32 [B, H, N] arrays written by the backward's first kernel:
 * -Delta (Delta_t = sum_d dO_td * O_td) and -lse_t * log2(e).
 */
S2ATTN_API size_t s2attn_bwd_workspace_bytes(int B, int H, int Hkv, int N, int D, int G);

/*
 * Backward.  Given the forward's inputs, its outputs o and lse, and the
 * upstream gradient dO, writes dq, dk, dv (fully overwritten; dk and dv are
 * summed over the query heads that share a kv-head).  Analytic gradient of
 * softmax attention: dP = dO V^T, dS = P * (dP - Delta), dQ = scale dS K,
 * dK = scale dS^T Q, dV = P^T dO, with P recomputed from lse.
 *   workspace: caller-owned device buffer of at least
 *   s2attn_bwd_workspace_bytes(...) bytes, 256-byte aligned; its status block
 *   is cleared by this call.
 */
S2ATTN_API int s2attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
               const void* dO, void* dq, void* dk, void* dv,
               int B, int H, int Hkv, int N, int D, int G,
               void* workspace, size_t workspace_bytes, s2attn_stream_t stream);

/*
 * Synchronises `stream`, then returns and clears the device status of the
 * most recent calls on this device (S2ATTN_OK, S2ATTN_ERR_DEVICE_TIMEOUT), or
 * S2ATTN_ERR_CUDA if the stream reports an error.  `workspace` is the buffer
 * given to s2attn_bwd, or NULL to read the forward's status block.
 */
S2ATTN_API int s2attn_device_status(void* workspace, s2attn_stream_t stream);

/* Static, human-readable name of a status code. */
S2ATTN_API const char* s2attn_status_string(int status);

/*
 * Backward for callers that cannot allocate device memory (no counterpart in
 * the papers: this is a deployment variant of s2attn_bwd).  Some callers have
 * no way to get a workspace: they run under another runtime's memory budget
 * without an allocator handle, inside plugin hosts that forbid cudaMalloc, or
 * must not allocate between set-up and graph capture.  This call computes
 * exactly what s2attn_bwd computes, with the same arguments minus the
 * workspace, and allocates nothing: its scratch (s2attn_bwd_workspace_bytes of
 * it) is a fixed 32 MiB device array inside the library, which every GPU that
 * loads the library holds until the process exits.  That limits it to
 * B * H * N <= 4194272 query rows (all five workload shapes fit); larger
 * shapes return S2ATTN_ERR_WORKSPACE without launching anything.
 *   - The first call on a device looks up the array's device address (with
 *     that device current) and caches it per device and context; make that
 *     first call before any stream capture.  After the device's context is
 *     destroyed and recreated (cudaDeviceReset), the next call looks the
 *     address up again, so it too should come before any stream capture.
 *   - All calls share the array and it keeps the last call's contents; each
 *     call rewrites what it reads.  Calls that overlap on the GPU (e.g. on two
 *     streams) race on it and must be serialised by the caller.
 *   - A bounded-wait timeout is recorded in the array's status block, which is
 *     not readable through s2attn_device_status; use s2attn_bwd when the
 *     device status is needed.
 */
S2ATTN_API int s2attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                  const float* lse, const void* dO, void* dq, void* dk, void* dv,
                                  int B, int H, int Hkv, int N, int D, int G,
                                  s2attn_stream_t stream);

/* ========================================================================
 * Test and benchmark hooks.  Not part of the operation: the test suite and
 * the benchmark use them to exercise the bounded waits, count launches and
 * time each kernel.  A caller of the attention needs none of them.
 * ======================================================================== */

/*
 * Self-test of the bounded wait every kernel uses: launches one block that
 * waits on an mbarrier nothing ever arrives at, with a `limit_ns` time limit,
 * and writes the resulting status code (S2ATTN_ERR_DEVICE_TIMEOUT expected)
 * to the device word *status_out.  No fault, trap or endless spin is involved.
 */
S2ATTN_API int s2attn_selftest_wait_timeout(uint32_t* status_out, uint64_t limit_ns, s2attn_stream_t stream);

/* Number of kernel launches the last s2attn_fwd / s2attn_bwd call made on this host thread. */
S2ATTN_API int s2attn_last_launch_count(void);

/*
 * Optional per-kernel timing for benchmarks (not part of the operation).
 * s2attn_profile_start creates 2 * max_launches CUDA events (no device memory)
 * and makes the following fwd/bwd calls on this host thread record one event
 * pair around each kernel they launch, up to max_launches launches.
 * s2attn_profile_stop turns recording off, waits for the recorded events and
 * writes per-launch durations (ms) and kernel ids (0 forward, 1 backward
 * preprocess, 2 backward dK/dV, 3 backward dQ) to caller arrays of
 * `capacity` entries (either may be NULL).  Returns the number of records, or
 * minus a status code.
 */
S2ATTN_API int s2attn_profile_start(int max_launches);
S2ATTN_API int s2attn_profile_stop(float* ms, int* kernel_ids, int capacity);

#ifdef __cplusplus
}
#endif

#endif /* S2ATTN_H_ */
