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
  S2ATTN_ERR_WORKSPACE = 6,      /* workspace missing or smaller than required */
  S2ATTN_ERR_DEVICE_BOUNDS = 7   /* debug build only: a kernel's computed index left its tensor (device status word) */
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
 * -Delta (Delta_t = sum_d dO_td * O_td) and -lse_t * log2(e); then what the
 * planned backward path keeps (s2attn_plan out[2]): for the split-dS path the
 * bf16 dS blocks (32 KB per 128 x 128 block, (H/Hkv) T (T+1)/2 blocks per
 * (batch, kv head, group), T = G/128) of out[5] such units at once, at most
 * 4 GiB unless the override asks for more; for the fused path an fp32
 * [B, H, N, D] accumulator for dq; nothing more for the split path.
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

/* ------------------------------------------------------------------------
 * Rotary position embedding with Position Interpolation before S2 attention.
 * LongQLoRA community post: LLaMA encodes positions with RoPE (section 02);
 * Position Interpolation shrinks RoPE's rotation angles to extend the context
 * from 4096 to 8192 tokens (section 04), and S2 attention then runs on the
 * rotated q and k.  Pair i of a head -- elements i and i + D/2 -- at token t
 * (original position) turns by  a(t, i) = t * pos_scale * rope_base^(-2i/D):
 *   y_i = x_i cos a - x_{i+D/2} sin a,   y_{i+D/2} = x_i sin a + x_{i+D/2} cos a.
 * pos_scale = L_train / L_target (0.5 for 4096 -> 8192; 1 is plain RoPE);
 * rope_base is the frequency base (10000 for LLaMA2).  v is not rotated.
 * ------------------------------------------------------------------------ */

/* Bytes of the rotary table for N positions at head dim D (0 if unsupported). */
S2ATTN_API size_t s2attn_rope_table_bytes(int N, int D);

/*
 * Fills `table` (device, caller-owned, s2attn_rope_table_bytes bytes, 16-byte
 * aligned) with fp32 (cos a, sin a) pairs, [N][D/2][2].  The angles are
 * formed and reduced in fp64 (at 100K tokens they reach ~1e5 radians).  The
 * table depends only on (N, D, pos_scale, rope_base): build it once and reuse
 * it across layers and steps.  D in {64, 128}, pos_scale > 0, rope_base > 1.
 */
S2ATTN_API int s2attn_rope_table(float* table, int N, int D, double pos_scale, double rope_base,
                                 s2attn_stream_t stream);

/*
 * out = x rotated by the table (by the opposite angles when `inverse` != 0,
 * which is the backward of the rotation).  x, out: bf16 [B, N, heads, D]
 * device buffers; out == x is allowed (in place).
 */
S2ATTN_API int s2attn_rope_apply(const void* x, void* out, const float* table, int B, int N, int heads, int D,
                                 int inverse, s2attn_stream_t stream);

/*
 * Forward of S2 attention on rotated inputs: q_rot = rotate(q), k_rot =
 * rotate(k) (caller buffers shaped like q and k, kept for the backward, not
 * aliasing q, k or each other), then o, lse = S2Attn(q_rot, k_rot, v) exactly
 * as s2attn_fwd.  Three launches.
 */
S2ATTN_API int s2attn_fwd_rope(const void* q, const void* k, const void* v, void* o, float* lse, void* q_rot,
                               void* k_rot, const float* table, int B, int H, int Hkv, int N, int D, int G,
                               s2attn_stream_t stream);

/*
 * Backward of s2attn_fwd_rope: takes the rotated q_rot, k_rot it produced and
 * writes the gradients with respect to the UNROTATED q and k (and v):
 * dq = rotate^-1(dq_rot), dk = rotate^-1(dk_rot).  On the fused backward path
 * (head dim 128) the back-rotation happens inside the dq conversion and the
 * dK epilogue; on the split path two in-place rotation passes follow.  The
 * workspace is that of s2attn_bwd (s2attn_bwd_workspace_bytes).
 */
S2ATTN_API int s2attn_bwd_rope(const void* q_rot, const void* k_rot, const void* v, const void* o,
                               const float* lse, const void* dO, void* dq, void* dk, void* dv, const float* table,
                               int B, int H, int Hkv, int N, int D, int G, void* workspace, size_t workspace_bytes,
                               s2attn_stream_t stream);

/* ------------------------------------------------------------------------
 * Chunk-wise attention over detached earlier keys (segment mode).  HGA digest
 * (arXiv 2607.15105): segment-wise backpropagation -- only the active segment
 * stays differentiable, older KV is detached and kept in another memory tier;
 * SeCO / SpaCO digest (arXiv 2505.16710): each chunk of a long input builds
 * its own graph and backpropagates locally.  The N query rows of the active
 * chunk are the last N rows of a sequence whose keys k, v hold Nk rows
 * (bf16 [B, Nk, Hkv, D]); with causal != 0 query row i attends keys
 * [0, Nk - N + i] (all earlier keys and its own chunk causally), with
 * causal == 0 every one of the Nk keys (a detached segment processed as a
 * piece of its own).  Dense causal softmax attention, no grouping or shift,
 * scale 1/sqrt(D); N and Nk multiples of 128; D in {64, 128}.
 * ------------------------------------------------------------------------ */

/* o bf16 [B, N, H, D], lse fp32 [B, H, N] of the segment attention. */
S2ATTN_API int s2attn_seg_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                              int Hkv, int N, int Nk, int D, int causal, s2attn_stream_t stream);

/* Workspace bytes of s2attn_seg_bwd (status block, Delta, lse*log2(e)). */
S2ATTN_API size_t s2attn_seg_bwd_workspace_bytes(int B, int H, int Hkv, int N, int Nk, int D);

/*
 * Backward of the segment attention given the FINAL o and lse of the chunk's
 * rows (after any lse merge of pieces): dq [B, N, H, D] through every key the
 * rows attend; with causal != 0 also dk, dv [B, N, Hkv, D] of the chunk's own
 * keys (the last N key rows; the earlier keys are detached and get no
 * gradient); with causal == 0 dk and dv must be NULL (dq only).
 * dq_accumulate != 0 adds the result to dq (summing the pieces of a query's
 * keys).  Split kernels: preprocess, dK/dV (causal only), dQ.
 */
S2ATTN_API int s2attn_seg_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                              const void* dO, void* dq, void* dk, void* dv, int B, int H, int Hkv, int N, int Nk,
                              int D, int causal, int dq_accumulate, void* workspace, size_t workspace_bytes,
                              s2attn_stream_t stream);

/*
 * Softmax attention over two disjoint key sets from the two pieces' results:
 * lse = log(exp(lse_a) + exp(lse_b)), o = exp(lse_a - lse) o_a + exp(lse_b - lse) o_b
 * (o_* bf16 [B, N, H, D], lse_* fp32 [B, H, N]; a piece with lse = -inf
 * counts for nothing).  o may be o_a and lse may be lse_a (in place).
 */
S2ATTN_API int s2attn_lse_merge(const void* o_a, const float* lse_a, const void* o_b, const float* lse_b, void* o,
                                float* lse, int B, int H, int N, int D, s2attn_stream_t stream);

/* ------------------------------------------------------------------------
 * HGA-style block-sparse attention over gathered history (HGA digest, arXiv
 * 2607.15105: each query block loads a bounded set of exact historical tokens;
 * only the active segment stays differentiable).  The sequence is cut into
 * segments of G rows (G % 256 == 0, N % G == 0; no head is shifted); a query
 * row attends its own segment's keys causally plus the historical key tiles
 * listed for its 256-row query block: hist is a device int32 [B, N/256, S]
 * array of 128-row key tile indices (tile e = key rows [128 e, 128 e + 128)),
 * shared by all heads.  A block uses its leading entries that name a tile of
 * an EARLIER segment (0 <= e < segment start / 128); the first other entry
 * (e.g. -1) ends its list.  Tensors, scale and lse as in s2attn_fwd.
 * ------------------------------------------------------------------------ */
S2ATTN_API int s2attn_hga_fwd(const void* q, const void* k, const void* v, void* o, float* lse, const int* hist,
                              int S, int B, int H, int Hkv, int N, int D, int G, s2attn_stream_t stream);

/* Workspace bytes of s2attn_hga_bwd. */
S2ATTN_API size_t s2attn_hga_bwd_workspace_bytes(int B, int H, int Hkv, int N, int D, int G);

/*
 * Backward of s2attn_hga_fwd: dq through every key a row attends; dk, dv
 * through the local (same-segment) attention only -- the historical keys are
 * detached.  Split kernels (preprocess, dK/dV, dQ over the listed tiles too).
 */
S2ATTN_API int s2attn_hga_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                              const void* dO, void* dq, void* dk, void* dv, const int* hist, int S, int B, int H,
                              int Hkv, int N, int D, int G, void* workspace, size_t workspace_bytes,
                              s2attn_stream_t stream);

/* ------------------------------------------------------------------------
 * QKV projection from 4-bit NormalFloat weights with double quantization
 * (LongQLoRA community post, section 03 Method, QLoRA: frozen weights in 4-bit
 * NF4, their quantization constants quantized again; section 04: the whole
 * model is quantized so, and S2 attention takes its q, k, v from these
 * projections).
 *
 * W is the [Nout, K] weight of the fused projection, Nout = (H + 2 Hkv) D:
 * rows [0, H D) produce q, [H D, (H + Hkv) D) k, the rest v; K is the model
 * width.  Its storage (all device memory, caller-owned, read only):
 *   codes        uint8 [Nout, K/2]: the 4-bit code of element 2j of a row in
 *                the low nibble of byte j, of element 2j+1 in the high nibble;
 *   scale_codes  int8 [Nout * K/64]: the first-level scale of block (n, kb)
 *                -- elements [64 kb, 64 kb + 64) of row n -- at n * K/64 + kb,
 *                as a code in [-127, 127];
 *   c2           fp32 [ceil(Nout * K/64 / 256)]: the second-level scale of
 *                first-level blocks [256 i, 256 i + 256) at i.
 * The dequantized weight is W'[n, k] = bf16(level[code] * s), s = code_s * c2
 * / 127, computed in fp32 and rounded to nearest even, with level[] the 16
 * NF4 values of s2attn_nf4_levels.
 * ------------------------------------------------------------------------ */

/* The 16 NF4 levels, ascending (level[c] for code c), as fp32 into the host
 * array levels[16]: standard normal quantiles normalised into [-1, 1] with an
 * exact zero (8 positive levels, 7 negative).  Host only. */
S2ATTN_API int s2attn_nf4_levels(float* levels);

/*
 * [q | k | v] = x W'^T with the dequantization fused into the tensor-core
 * GEMM (W' never goes to global memory).  x: bf16 [M, K] (M tokens, row
 * major, 16-byte aligned); q: bf16 [M, H D], k and v: bf16 [M, Hkv D], row
 * major -- i.e. [B, N, heads, D] with M = B N, the layout s2attn_fwd reads.
 * fp32 accumulation, bf16 results rounded to nearest even.  Requires
 * K % 64 == 0 and H D, Hkv D multiples of 128; codes, q, k, v 16-byte
 * aligned.
 * Returns a status code; a bounded-wait timeout inside the kernel is reported
 * by s2attn_device_status(NULL, stream).
 */
S2ATTN_API int s2attn_nf4_qkv(const void* x, const void* codes, const int8_t* scale_codes, const float* c2,
                              void* q, void* k, void* v, int M, int K, int H, int Hkv, int D,
                              s2attn_stream_t stream);

/*
 * The dequantized weight alone: w = W' as bf16 [rows, K] (16-byte aligned),
 * from codes [rows, K/2] (4-byte aligned), scale_codes and c2 laid out as
 * above with `rows` in place of Nout.  K % 64 == 0.  For callers that run
 * their own GEMM on W' (e.g. the input gradient x' = y' W').
 */
S2ATTN_API int s2attn_nf4_dequant(const void* codes, const int8_t* scale_codes, const float* c2, void* w,
                                  int rows, int K, s2attn_stream_t stream);

/*
 * Backward for callers that cannot allocate device memory (no counterpart in
 * the papers: this is a deployment variant of s2attn_bwd).  Some callers have
 * no way to get a workspace: they run under another runtime's memory budget
 * without an allocator handle, inside plugin hosts that forbid cudaMalloc, or
 * must not allocate between set-up and graph capture.  This call computes
 * the same gradients as s2attn_bwd, with the same arguments minus the
 * workspace, and allocates nothing.  It runs the split backward (preprocess,
 * dK/dV kernel, dQ kernel), whose scratch -- status block, Delta and
 * lse*log2(e), 256 + 2 * round_up(4 * B * H * N, 256) bytes -- is a fixed
 * 32 MiB device array inside the library, which every GPU that loads the
 * library holds until the process exits.  That limits it to
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

/*
 * 1 if this library is the debug build (libs2attn_debug.so, compiled with
 * S2ATTN_DEBUG_CHECKS): its kernels check every computed global index
 * against its tensor before the access, skip an access that falls outside
 * and record S2ATTN_ERR_DEVICE_BOUNDS with the site in the device status word
 * (read by s2attn_device_status).  0 for the default build, which has no
 * such checks.
 */
S2ATTN_API int s2attn_debug_checks(void);

/* Number of kernel launches the last s2attn_fwd / s2attn_bwd call made on this host thread. */
S2ATTN_API int s2attn_last_launch_count(void);

/*
 * Diagnosis of S2ATTN_ERR_CUDA: the last CUDA runtime error code behind one
 * on this host thread (or minus the driver's result when a TMA tensor map
 * could not be encoded; 0 if none), and a static description of such a code.
 */
S2ATTN_API int s2attn_last_cuda_error(void);
S2ATTN_API const char* s2attn_cuda_error_string(int err);

/*
 * Optional per-kernel timing for benchmarks (not part of the operation).
 * s2attn_profile_start creates 2 * max_launches CUDA events (no device memory)
 * and makes the following fwd/bwd calls on this host thread record one event
 * pair around each kernel they launch, up to max_launches launches.
 * s2attn_profile_stop turns recording off, waits for the recorded events and
 * writes per-launch durations (ms) and kernel ids (0 forward, 1 backward
 * preprocess, 2 backward dK/dV, 3 backward dQ, 4 fused backward, 5 its dq
 * conversion, 6 RoPE rotation, 7 NF4 QKV projection, 8 NF4 dequantization, 9
 * backward dQ from the stored dS) to caller arrays of
 * `capacity` entries (either may be NULL).  Returns the number of records, or
 * minus a status code.
 */
S2ATTN_API int s2attn_profile_start(int max_launches);
S2ATTN_API int s2attn_profile_stop(float* ms, int* kernel_ids, int capacity);

/*
 * The per-shape plan the library would use for a call with these arguments on
 * a device with num_sms SMs (with the override below applied): out[0] forward
 * work order (1 longest-first snake, 0 equal-work pairs), out[1] forward K/V
 * ring depth, out[2] backward path (2 split-dS: dQ from the dS blocks the
 * dK/dV kernel stores in the workspace; 0 split: dQ recomputes S and dP; 1
 * fused), out[3] split backward pipeline stages, out[4] forward key tile (128,
 * or 64 with double-buffered scores), out[5] on the split-dS path the dK/dV
 * units (batch x kv head x group) whose dS blocks the workspace holds at once
 * (all of them when they fit its 4 GiB budget; fewer, and the backward runs
 * its dK/dV work in ranges of pairs each followed by dQ for the units the
 * range completed), else 0; out[6] the dK/dV kernel's query tile (64: 64-row
 * sub-tiles; 128: 128-row tiles, whose S^T / dP^T UMMAs are twice as wide;
 * S2 attention calls only, the chunk-wise and HGA backwards take 64).  `out`
 * holds 7 ints.  Host only; returns a status code (shape validation as in
 * s2attn_fwd).
 */
S2ATTN_API int s2attn_plan(int B, int H, int Hkv, int N, int D, int G, int num_sms, int* out);

/*
 * Replaces the plan override (initially the S2ATTN_TILE environment
 * variable) that later calls in this process consult; NULL restores the
 * environment's value.  The override forces a variant the per-shape selection
 * would not pick, for tests and sweeps: a comma-separated list of key=value
 * items; keys bwd=split_ds|split|fused (backward path; fused exists for head dim 128),
 * ds_slots=N (N >= 2: the split-dS path's workspace holds dS of N dK/dV units),
 * bwd_qtile=64|128 (the dK/dV kernel's query tile),
 * fwd_order=snake|pairs (forward work order), fwd_bn=64|128 (forward key
 * tile), fwd_kv=N (forward K/V ring depth: with 128-key tiles 4 at head dim
 * 128, 4/6/8 at 64; with 64-key tiles 8 at head dim 128, 8/12 at 64), bwd_stages=N (dK/dV operand
 * stages: 2-4 at head dim 128, 3-4 at 64; the split path's dQ kernel takes at
 * most 3 at head dim 128), nf4_stages=4|5 and nf4_dq=8|12
 * (pipeline depth and dequantization warps of s2attn_nf4_qkv); values that do not exist for a call's head dim
 * are ignored.  s2attn_bwd_workspace_bytes answers for the
 * path in force when it is called.  Returns S2ATTN_OK.
 */
S2ATTN_API int s2attn_set_tile_override(const char* spec);

#ifdef __cplusplus
}
#endif

#endif /* S2ATTN_H_ */
