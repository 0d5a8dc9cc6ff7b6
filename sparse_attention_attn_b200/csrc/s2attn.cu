// Host side of the C ABI declared in include/s2attn.h: argument validation,
// TMA tensor-map encoding, kernel launches and status reporting.
//
// Nothing here allocates device memory at run time: the caller owns every
// buffer it passes.  The library's own device state is fixed at module load:
// the forward's status block and the scratch array of s2attn_bwd_noalloc,
// both file-scope __device__ arrays.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <mutex>
#include <string>
#include <vector>

#include "s2_common.cuh"
#include "s2_ptx.cuh"
#include "s2attn.h"

namespace s2 {
template <int D>
cudaError_t launch_fwd(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                       const FwdArgs&, int, cudaStream_t, int);
template <int D>
cudaError_t launch_fwd64(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                         const FwdArgs&, int, cudaStream_t, int);
template <int D>
cudaError_t launch_bwd(const BwdMaps&, const BwdPreArgs&, const BwdArgs&, int, cudaStream_t, int*, int);
template <int D>
cudaError_t launch_bwd_fused(const BwdMaps&, const BwdPreArgs&, const BwdArgs&, int, cudaStream_t, int*);
cudaError_t launch_rope_table(float* table, int N, int D, double pos_scale, double base, int num_sms,
                              cudaStream_t stream);
cudaError_t launch_rope_apply(const void* x, void* out, const float* table, int B, int N, int heads, int D,
                              int inverse, int num_sms, cudaStream_t stream);
cudaError_t launch_lse_merge(const void* oa, const float* la, const void* ob, const float* lb, void* o, float* lse,
                             int B, int H, int N, int D, int num_sms, cudaStream_t stream);
}  // namespace s2

namespace {

using namespace s2;

__device__ uint32_t g_fwd_status[4];  // [0] error code, [1] where

thread_local int g_last_launches = 0;
// The last CUDA runtime error (or -(driver result) of a tensor-map encoding)
// behind an S2ATTN_ERR_CUDA on this host thread, for diagnosis.
thread_local int g_last_cuda_error = 0;

constexpr size_t kStatusBytes = 256;

// Backward paths.  Split: preprocess, dK/dV kernel, dQ kernel (recomputes S
// and dP).  Fused (head dim 128): preprocess, one kernel for dK, dV and the
// dQ partials (reduced into an fp32 accumulator in the workspace), dq
// conversion.
enum BwdPath : int { kBwdSplit = 0, kBwdFused = 1, kBwdSplitDs = 2 };

// The split-dS path stores the dS blocks (32 KB per (query tile, kv tile <=
// it) of each (batch, head, group)) in the workspace, within this budget: all
// of them when they fit, else those of as many dK/dV units (batch x kv head x
// group, with its query heads) as fit, the backward then running in ranges.
constexpr double kDsBudgetBytes = 4.0 * 1024 * 1024 * 1024;

// dS blocks of one dK/dV unit: (H/Hkv) T (T+1) / 2, T = G/128.
long long ds_unit_blocks(int H, int Hkv, int G) {
  const long long T = G / kTile;
  return static_cast<long long>(H / Hkv) * (T * (T + 1) / 2);
}

// dK/dV units whose dS the workspace holds at once: every unit if they fit
// the budget, else as many as fit if that is at least 2 (each range of the
// backward then completes at least one unit), else 0 (no split-dS plan).
// `want` > 0 (a plan override) asks for that many instead, from 2 up.
int ds_slots_for(int B, int H, int Hkv, int N, int G, int want = 0) {
  const long long units = static_cast<long long>(B) * Hkv * (N / G);
  const double unit_bytes = static_cast<double>(ds_unit_blocks(H, Hkv, G)) * kTile * kTile * 2;
  long long fit = static_cast<long long>(kDsBudgetBytes / unit_bytes);
  if (want >= 2) fit = want;
  if (fit >= units) return static_cast<int>(units);
  return fit >= 2 ? static_cast<int>(fit) : 0;
}


typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Per-device facts cached on first use: is it sm_100, how many SMs.
struct DeviceInfo {
  bool ok = false;
  int sms = 0;
};

bool device_info(DeviceInfo* out) {
  static std::mutex mu;
  static DeviceInfo cache[64];
  static bool known[64] = {};
  int dev = 0;
  cudaError_t ge = cudaGetDevice(&dev);
  // bind the device's primary context to this host thread: the TMA
  // descriptors are encoded through the driver API, which needs a current
  // context, and a thread that has made no runtime call yet (e.g. an autograd
  // worker running a backward) may have none
  if (ge == cudaSuccess) ge = cudaSetDevice(dev);
  if (ge != cudaSuccess || dev < 0 || dev >= 64) {
    g_last_cuda_error = static_cast<int>(ge);
    return false;
  }
  std::lock_guard<std::mutex> lk(mu);
  if (!known[dev]) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return false;
    cache[dev].ok = (major == 10 && minor == 0);
    cache[dev].sms = sms;
    known[dev] = true;
  }
  *out = cache[dev];
  return true;
}

unsigned long long wait_limit_ns() {
  static unsigned long long v = [] {
    const char* e = std::getenv("S2ATTN_WAIT_LIMIT_MS");
    long long ms = e ? std::atoll(e) : 2000;
    if (ms <= 0) ms = 2000;
    return static_cast<unsigned long long>(ms) * 1000000ull;
  }();
  return v;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape rules shared by forward and backward.  Pure host logic: no CUDA call.
int validate_shape(int B, int H, int Hkv, int N, int D, int G, bool shifted = true) {
  if (B <= 0 || H <= 0 || Hkv <= 0 || N <= 0 || D <= 0 || G <= 0) return S2ATTN_ERR_INVALID_ARG;
  if (H % Hkv != 0 || G > N || N % G != 0) return S2ATTN_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return S2ATTN_ERR_UNSUPPORTED;
  if (N % kTile != 0 || G % kTile != 0) return S2ATTN_ERR_UNSUPPORTED;
  if (G < N && shifted) {  // the shifted half of the heads takes whole kv-head groups
    if (G % (2 * kTile) != 0) return S2ATTN_ERR_UNSUPPORTED;
    if ((H / 2) % (H / Hkv) != 0) return S2ATTN_ERR_UNSUPPORTED;
  }
  // grid sizes and element offsets stay well inside 32/64-bit ranges
  const long long q_tiles = static_cast<long long>(B) * H * (N / kTile);
  if (q_tiles > (1LL << 30)) return S2ATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(N) * H * D >= (1LL << 40)) return S2ATTN_ERR_UNSUPPORTED;
  return S2ATTN_OK;
}

Dims make_dims(int B, int H, int Hkv, int N, int D, int G) {
  Dims d;
  d.B = B;
  d.H = H;
  d.Hkv = Hkv;
  d.N = N;
  d.D = D;
  d.G = G;
  d.rep = H / Hkv;
  d.n_groups = N / G;
  d.tiles = G / kTile;
  d.Nk = N;
  d.qoff_t = 0;
  d.causal = 1;
  d.noshift = 0;
  return d;
}

// Segment mode (chunk-wise attention): N query rows over Nk key rows, one
// group, no shift; causal: query row i sees keys [0, Nk - N + i].
int validate_segment(int B, int H, int Hkv, int N, int Nk, int D, int causal) {
  if (B <= 0 || H <= 0 || Hkv <= 0 || N <= 0 || Nk <= 0 || D <= 0) return S2ATTN_ERR_INVALID_ARG;
  if (H % Hkv != 0 || (causal && Nk < N)) return S2ATTN_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return S2ATTN_ERR_UNSUPPORTED;
  if (N % kTile != 0 || Nk % kTile != 0) return S2ATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H * (N / kTile) > (1LL << 30)) return S2ATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(Nk) * H * D >= (1LL << 40)) return S2ATTN_ERR_UNSUPPORTED;
  return S2ATTN_OK;
}

Dims make_segment_dims(int B, int H, int Hkv, int N, int Nk, int D, int causal) {
  Dims d = make_dims(B, H, Hkv, N, D, N);  // one group of N rows, no shift
  d.Nk = Nk;
  d.qoff_t = causal ? (Nk - N) / kTile : 0;
  d.causal = causal ? 1 : 0;
  return d;
}

// ---------------------------------------------------------------- plan override
// A plan override string ("key=value,..."), used to time or test a variant
// that the per-shape selection would not pick.  It starts from the
// S2ATTN_TILE environment variable and can be replaced at run time by the
// s2attn_set_tile_override test hook.  Keys: bwd=split_ds|split|fused, ds_slots=N, bwd_qtile=64|128,
// fwd_order=snake|pairs, fwd_bn=64|128, fwd_kv=N, bwd_stages=N, nf4_stages=4|5, nf4_dq=8|12.  Unknown
// keys and values are ignored.
std::mutex g_override_mu;
std::string g_override;
bool g_override_init = false;

std::string tile_override() {
  std::lock_guard<std::mutex> lk(g_override_mu);
  if (!g_override_init) {
    const char* e = std::getenv("S2ATTN_TILE");
    g_override = e ? e : "";
    g_override_init = true;
  }
  return g_override;
}

// Value of `key` in the override string, or "" if absent.
std::string override_value(const std::string& spec, const char* key) {
  const std::string k = std::string(key) + "=";
  size_t pos = 0;
  while (pos < spec.size()) {
    size_t end = spec.find(',', pos);
    if (end == std::string::npos) end = spec.size();
    const std::string item = spec.substr(pos, end - pos);
    if (item.compare(0, k.size(), k) == 0) return item.substr(k.size());
    pos = end + 1;
  }
  return "";
}

// ---------------------------------------------------------------- per-shape plan
// The kernel variant and pipeline depths for one call, chosen from the shape
// (D, G, N, H, Hkv, B) and the SM count; the table below follows the sweep
// recorded under profiles/ (every variant timed on the five workload shapes).
struct Plan {
  int fwd_snake;     // forward work order: 1 snake (longest first), 0 equal-work pairs
  int fwd_bn;        // forward key tile: 128 (s2_fwd.cu) or 64 with double-buffered scores (s2_fwd64.cu)
  int fwd_kv_slots;  // forward K/V ring depth: 128-key tiles 4 (head dim 128), 4/6/8 (head dim 64);
                     // 64-key tiles 8 (head dim 128), 8/12 (head dim 64)
  int bwd_path;      // kBwdSplitDs, kBwdSplit, or kBwdFused (head dim 128 only)
  int bwd_stages;    // dK/dV operand stages: 2-4 (head dim 128; the split dQ kernel at most 3), 3-4 (head dim 64)
  int ds_slots;      // split-dS path: dK/dV units whose dS the workspace holds (see ds_slots_for)
  int bwd_qtile;     // dK/dV query tile: 64 (sub-tiles, s2_bwd.cu) or 128 (s2_bwd_kv128.cu)
};

bool valid_kv_slots(int D, int bn, int v) {
  if (bn == 64) return D == 128 ? v == 8 : (v == 8 || v == 12);
  return D == 128 ? v == 4 : (v == 4 || v == 6 || v == 8);
}
bool valid_bwd_stages(int D, int v) { return D == 128 ? (v >= 2 && v <= 4) : (v == 3 || v == 4); }

Plan select_plan(int B, int H, int Hkv, int N, int D, int G, int sms) {
  (void)H;
  (void)G;
  (void)sms;
  Plan p;
  // The snake order balances the CTAs best but spreads the units over all of
  // them at once, so it is taken while K and V together stay within about
  // twice the L2 (126 MB): beyond that the pairs order keeps the readers of a
  // K/V tile running together.
  const double kv_bytes = 2.0 * B * N * Hkv * D * 2.0;
  p.fwd_snake = kv_bytes <= 256.0 * 1024 * 1024 ? 1 : 0;
  p.fwd_bn = 128;
  p.fwd_kv_slots = D == 128 ? 4 : 8;
  // dQ from the dS the dK/dV kernel stores (five GEMM-units instead of
  // seven) while the dS blocks fit the budget, else the split path that
  // recomputes S and dP for dQ; the fused path measured slower than both and
  // stays selectable
  p.ds_slots = ds_slots_for(B, H, Hkv, N, G);
  p.bwd_path = p.ds_slots > 0 ? kBwdSplitDs : kBwdSplit;
  p.bwd_stages = 3;
  p.bwd_qtile = 64;
  // the override, where it names a variant that exists for this head dim
  const std::string spec = tile_override();
  const std::string order = override_value(spec, "fwd_order");
  if (order == "snake") p.fwd_snake = 1;
  if (order == "pairs") p.fwd_snake = 0;
  const std::string bn = override_value(spec, "fwd_bn");
  if (bn == "64" && p.fwd_bn != 64) {
    p.fwd_bn = 64;
    p.fwd_kv_slots = 8;
  }
  if (bn == "128" && p.fwd_bn != 128) {
    p.fwd_bn = 128;
    p.fwd_kv_slots = D == 128 ? 4 : 8;
  }
  const std::string kv = override_value(spec, "fwd_kv");
  if (!kv.empty() && valid_kv_slots(D, p.fwd_bn, std::atoi(kv.c_str()))) p.fwd_kv_slots = std::atoi(kv.c_str());
  const std::string path = override_value(spec, "bwd");
  if (path == "split") p.bwd_path = kBwdSplit;
  const std::string slots = override_value(spec, "ds_slots");
  if (!slots.empty() && std::atoi(slots.c_str()) >= 2) p.ds_slots = ds_slots_for(B, H, Hkv, N, G, std::atoi(slots.c_str()));
  if (path == "split_ds" && p.ds_slots == 0) p.ds_slots = ds_slots_for(B, H, Hkv, N, G, 2);
  if (path == "split_ds") p.bwd_path = kBwdSplitDs;
  if (path == "fused" && D == 128) p.bwd_path = kBwdFused;
  const std::string qt = override_value(spec, "bwd_qtile");
  if (qt == "64") p.bwd_qtile = 64;
  if (qt == "128") p.bwd_qtile = 128;
  const std::string st = override_value(spec, "bwd_stages");
  if (!st.empty() && valid_bwd_stages(D, std::atoi(st.c_str()))) p.bwd_stages = std::atoi(st.c_str());
  return p;
}

// Forward work order (see FwdSched).
FwdSched make_fwd_sched(const Dims& d, int snake) {
  FwdSched s;
  s.units = d.B * d.H * d.n_groups;
  s.Ti = (d.tiles + 1) / 2;
  s.ppu = (s.Ti + 1) / 2;
  s.snake = snake;
  s.n = s.snake ? s.units * s.Ti : s.units * s.ppu;
  return s;
}

// 4-D view {D, heads, N, B} of a bf16 [B, N, heads, D] tensor; box = one
// box_rows x 64-column slab, 128-byte swizzle (the UMMA operand layout).
bool make_map(CUtensorMap* m, const void* base, int B, int N, int heads, int D, int box_rows = kTile) {
  EncodeTiledFn enc = get_encode();
  if (!enc) {
    g_last_cuda_error = -1;
    return false;
  }
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(heads),
                        static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(heads) * D * 2,
                           static_cast<cuuint64_t>(N) * heads * D * 2};
  cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) g_last_cuda_error = -static_cast<int>(r);
  return r == CUDA_SUCCESS;
}

// 2-D tiled view {inner, outer} of a row-major array with `row_bytes` between rows.
bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                 uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  EncodeTiledFn enc = get_encode();
  if (!enc) {
    g_last_cuda_error = -1;
    return false;
  }
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  const CUresult r = enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) g_last_cuda_error = -static_cast<int>(r);
  return r == CUDA_SUCCESS;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

size_t rowstat_bytes(int B, int H, int N) {
  return round_up(static_cast<size_t>(B) * H * N * sizeof(float), 256);
}

// Workspace: status block, -Delta, -lse*log2(e); for the fused path the fp32
// [B, H, N, D] dQ accumulator; for the split-dS path `ds_blocks` dS blocks.
size_t workspace_bytes_for(int path, int B, int H, int N, int D, long long ds_blocks = 0) {
  size_t n = kStatusBytes + 2 * rowstat_bytes(B, H, N);
  if (path == kBwdFused) n += round_up(static_cast<size_t>(B) * H * N * D * sizeof(float), 256);
  if (path == kBwdSplitDs) n += static_cast<size_t>(ds_blocks) * kTile * kTile * 2;
  return n;
}

__global__ void s2_selftest_wait_kernel(uint32_t* status, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    status[0] = 0;
    status[1] = 0;
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    WaitCtx wc{&abort_flag, status, limit_ns};
    mbar_wait(smem_u32(&bar), 0, wc, 999);  // nothing ever arrives: runs out, records, returns
  }
}

// Per-host-thread launch timing.  Events are created once by
// s2attn_profile_start and reused; no device memory is involved.
struct ProfRecord {
  cudaEvent_t start, stop;
  int kernel;
};
struct ProfState {
  bool on = false;
  std::vector<ProfRecord> recs;
  size_t used = 0;
};
thread_local ProfState g_prof;

// The forward of a validated shape (S2 attention or a segment).
int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, const Dims& dims,
             s2attn_stream_t stream, HgaList hist = HgaList()) {
  const int B = dims.B, H = dims.H, Hkv = dims.Hkv, N = dims.N, D = dims.D, G = dims.G;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return S2ATTN_ERR_MISALIGNED;
  DeviceInfo info;
  if (!device_info(&info)) return S2ATTN_ERR_CUDA;
  if (!info.ok) return S2ATTN_ERR_UNSUPPORTED;
  const Plan plan = select_plan(B, H, Hkv, N, D, G, info.sms);
  CUtensorMap tq, tk, tv, to;
  if (!make_map(&tq, q, B, N, H, D) || !make_map(&tk, k, B, dims.Nk, Hkv, D, plan.fwd_bn) ||
      !make_map(&tv, v, B, dims.Nk, Hkv, D, plan.fwd_bn) || !make_map(&to, o, B, N, H, D, 32))
    return S2ATTN_ERR_CUDA;
  FwdArgs a;
  a.d = dims;
  a.hist = hist;
  a.sched = make_fwd_sched(a.d, plan.fwd_snake);
  a.scale_log2 = static_cast<float>(1.4426950408889634 / __builtin_sqrt(static_cast<double>(D)));
  a.lse = lse;  // o is written through its TMA map
  void* status = nullptr;
  const cudaError_t se = cudaGetSymbolAddress(&status, g_fwd_status);
  if (se != cudaSuccess) {
    g_last_cuda_error = static_cast<int>(se);
    return S2ATTN_ERR_CUDA;
  }
  a.status = static_cast<uint32_t*>(status);
  a.wait_limit_ns = wait_limit_ns();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (plan.fwd_bn == 64)
    e = (D == 64) ? launch_fwd64<64>(tq, tk, tv, to, a, info.sms, s, plan.fwd_kv_slots)
                  : launch_fwd64<128>(tq, tk, tv, to, a, info.sms, s, plan.fwd_kv_slots);
  else
    e = (D == 64) ? launch_fwd<64>(tq, tk, tv, to, a, info.sms, s, plan.fwd_kv_slots)
                  : launch_fwd<128>(tq, tk, tv, to, a, info.sms, s, plan.fwd_kv_slots);
  if (e != cudaSuccess) {
    g_last_cuda_error = static_cast<int>(e);
    return S2ATTN_ERR_CUDA;
  }
  g_last_launches = 1;
  return S2ATTN_OK;
}

}  // namespace

namespace s2 {
void prof_before(cudaStream_t stream, int kernel_id) {
  if (!g_prof.on || g_prof.used >= g_prof.recs.size()) return;
  ProfRecord& r = g_prof.recs[g_prof.used];
  r.kernel = kernel_id;
  cudaEventRecord(r.start, stream);
}
void prof_after(cudaStream_t stream) {
  if (!g_prof.on || g_prof.used >= g_prof.recs.size()) return;
  cudaEventRecord(g_prof.recs[g_prof.used].stop, stream);
  ++g_prof.used;
}
}  // namespace s2

extern "C" {

int s2attn_profile_start(int max_launches) {
  if (max_launches <= 0 || max_launches > (1 << 20)) return S2ATTN_ERR_INVALID_ARG;
  for (ProfRecord& r : g_prof.recs) {
    cudaEventDestroy(r.start);
    cudaEventDestroy(r.stop);
  }
  g_prof.recs.clear();
  g_prof.used = 0;
  g_prof.on = false;
  for (int i = 0; i < max_launches; ++i) {
    ProfRecord r{nullptr, nullptr, -1};
    if (cudaEventCreate(&r.start) != cudaSuccess || cudaEventCreate(&r.stop) != cudaSuccess)
      return S2ATTN_ERR_CUDA;
    g_prof.recs.push_back(r);
  }
  g_prof.on = true;
  return S2ATTN_OK;
}

int s2attn_profile_stop(float* ms, int* kernel_ids, int capacity) {
  if (!g_prof.on) return 0;
  g_prof.on = false;
  const int n = static_cast<int>(g_prof.used);
  int out = 0;
  for (int i = 0; i < n && out < capacity; ++i) {
    float t = 0.f;
    if (cudaEventSynchronize(g_prof.recs[i].stop) != cudaSuccess ||
        cudaEventElapsedTime(&t, g_prof.recs[i].start, g_prof.recs[i].stop) != cudaSuccess)
      return -S2ATTN_ERR_CUDA;
    if (ms) ms[out] = t;
    if (kernel_ids) kernel_ids[out] = g_prof.recs[i].kernel;
    ++out;
  }
  g_prof.used = 0;
  return out;
}


const char* s2attn_status_string(int status) {
  switch (status) {
    case S2ATTN_OK: return "S2ATTN_OK";
    case S2ATTN_ERR_INVALID_ARG: return "S2ATTN_ERR_INVALID_ARG";
    case S2ATTN_ERR_UNSUPPORTED: return "S2ATTN_ERR_UNSUPPORTED";
    case S2ATTN_ERR_MISALIGNED: return "S2ATTN_ERR_MISALIGNED";
    case S2ATTN_ERR_CUDA: return "S2ATTN_ERR_CUDA";
    case S2ATTN_ERR_DEVICE_TIMEOUT: return "S2ATTN_ERR_DEVICE_TIMEOUT";
    case S2ATTN_ERR_WORKSPACE: return "S2ATTN_ERR_WORKSPACE";
    case S2ATTN_ERR_DEVICE_BOUNDS: return "S2ATTN_ERR_DEVICE_BOUNDS";
    default: return "S2ATTN_UNKNOWN_STATUS";
  }
}

int s2attn_last_launch_count(void) { return g_last_launches; }

int s2attn_debug_checks(void) {
#ifdef S2ATTN_DEBUG_CHECKS
  return 1;
#else
  return 0;
#endif
}

int s2attn_last_cuda_error(void) { return g_last_cuda_error; }

const char* s2attn_cuda_error_string(int err) {
  if (err < 0) return "tensor-map encoding failed (minus the driver result)";
  return cudaGetErrorString(static_cast<cudaError_t>(err));
}

size_t s2attn_bwd_workspace_bytes(int B, int H, int Hkv, int N, int D, int G) {
  if (validate_shape(B, H, Hkv, N, D, G) != S2ATTN_OK) return 0;
  const Plan p = select_plan(B, H, Hkv, N, D, G, 0);
  return workspace_bytes_for(p.bwd_path, B, H, N, D, p.ds_slots * ds_unit_blocks(H, Hkv, G));
}

int s2attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
               int Hkv, int N, int D, int G, s2attn_stream_t stream) {
  g_last_launches = 0;
  if (!q || !k || !v || !o || !lse) return S2ATTN_ERR_INVALID_ARG;
  int st = validate_shape(B, H, Hkv, N, D, G);
  if (st != S2ATTN_OK) return st;
  return fwd_impl(q, k, v, o, lse, make_dims(B, H, Hkv, N, D, G), stream);
}

int s2attn_seg_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv,
                   int N, int Nk, int D, int causal, s2attn_stream_t stream) {
  g_last_launches = 0;
  if (!q || !k || !v || !o || !lse) return S2ATTN_ERR_INVALID_ARG;
  int st = validate_segment(B, H, Hkv, N, Nk, D, causal);
  if (st != S2ATTN_OK) return st;
  return fwd_impl(q, k, v, o, lse, make_segment_dims(B, H, Hkv, N, Nk, D, causal), stream);
}
}  // extern "C"

namespace {
// The backward on `path` (kBwdSplitDs, kBwdSplit or kBwdFused); ds_slots: the
// split-dS path's dK/dV units of dS in the workspace (ds_slots_for); qtile:
// the dK/dV kernel's query tile (128 for S2 attention only; 64 otherwise).  `seg`: segment-mode
// dimensions (chunk-wise attention; split path only), or null for S2
// attention of (B, H, Hkv, N, D, G).  Segment mode with causal = 0 computes dq
// only (dk = dv = null: a detached key segment); dq_accumulate adds the
// result to dq.
int bwd_impl(int path, int stages, int ds_slots, int qtile, const void* q, const void* k, const void* v, const void* o, const float* lse,
             const void* dO, void* dq, void* dk, void* dv, int B, int H, int Hkv, int N, int D, int G,
             void* workspace, size_t workspace_bytes, s2attn_stream_t stream, const float* rope = nullptr,
             const Dims* seg = nullptr, int dq_accumulate = 0, HgaList hist = HgaList()) {
  g_last_launches = 0;
  const bool dq_only = seg != nullptr && !seg->causal;
  if (!q || !k || !v || !o || !lse || !dO || !dq) return S2ATTN_ERR_INVALID_ARG;
  if (dq_only ? (dk != nullptr || dv != nullptr) : (!dk || !dv)) return S2ATTN_ERR_INVALID_ARG;
  if (seg == nullptr) {
    const int st = validate_shape(B, H, Hkv, N, D, G);
    if (st != S2ATTN_OK) return st;
  }
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      !aligned16(dO) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return S2ATTN_ERR_MISALIGNED;
  // segment and HGA modes take the split path (the dQ kernel walks their extra keys)
  if (seg != nullptr && path == kBwdSplitDs) path = kBwdSplit;
  if (path == kBwdSplitDs && ds_slots < 2 && ds_slots < B * Hkv * (N / G)) path = kBwdSplit;
  const long long ds_blocks = path == kBwdSplitDs ? ds_slots * ds_unit_blocks(H, Hkv, G) : 0;
  const size_t need = workspace_bytes_for(path, B, H, N, D, ds_blocks);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return S2ATTN_ERR_WORKSPACE;
  DeviceInfo info;
  if (!device_info(&info)) return S2ATTN_ERR_CUDA;
  if (!info.ok) return S2ATTN_ERR_UNSUPPORTED;
  const Dims d = seg ? *seg : make_dims(B, H, Hkv, N, D, G);
  const int Nk = d.Nk;
  BwdMaps maps;
  if (!make_map(&maps.q128, q, B, N, H, D) || !make_map(&maps.k128, k, B, Nk, Hkv, D) ||
      !make_map(&maps.v128, v, B, Nk, Hkv, D) || !make_map(&maps.g128, dO, B, N, H, D) ||
      !make_map(&maps.q64, q, B, N, H, D, 64) || !make_map(&maps.k64, k, B, Nk, Hkv, D, 64) ||
      !make_map(&maps.v64, v, B, Nk, Hkv, D, 64) || !make_map(&maps.g64, dO, B, N, H, D, 64))
    return S2ATTN_ERR_CUDA;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  float* ndelta = reinterpret_cast<float*>(ws + kStatusBytes);
  float* nlse2 = reinterpret_cast<float*>(ws + kStatusBytes + rowstat_bytes(B, H, N));
  float* dqacc = path == kBwdFused ? reinterpret_cast<float*>(ws + kStatusBytes + 2 * rowstat_bytes(B, H, N))
                                   : nullptr;
  __nv_bfloat16* ds = path == kBwdSplitDs
                          ? reinterpret_cast<__nv_bfloat16*>(ws + kStatusBytes + 2 * rowstat_bytes(B, H, N))
                          : nullptr;
  if (ds != nullptr &&
      (!make_map_2d(&maps.ds, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, ds, 32, static_cast<uint64_t>(ds_blocks) * 4 * kTile,
                    64, 32, 2 * kTile, CU_TENSOR_MAP_SWIZZLE_64B) ||
       !make_map(&maps.dq32, dq, B, N, H, D, 32)))
    return S2ATTN_ERR_CUDA;
  BwdPreArgs pre;
  pre.d = d;
  pre.o = o;
  pre.dO = dO;
  pre.lse = lse;
  pre.ndelta = ndelta;
  pre.nlse2 = nlse2;
  pre.dqacc = dqacc;
  pre.status = status;
  BwdArgs a;
  a.d = d;
  a.hist = hist;
  a.kv_sched = make_pair_sched(B * Hkv * d.n_groups, d.tiles);
  a.q_sched = make_pair_sched(B * H * d.n_groups, d.tiles);
  a.scale = static_cast<float>(1.0 / __builtin_sqrt(static_cast<double>(D)));
  a.scale_log2 = static_cast<float>(1.4426950408889634 / __builtin_sqrt(static_cast<double>(D)));
  a.ndelta = ndelta;
  a.nlse2 = nlse2;
  a.dq = dq;
  a.dq_accumulate = dq_accumulate ? 1 : 0;
  a.no_dkdv = dq_only ? 1 : 0;
  a.dqacc = dqacc;
  a.dk = dk;
  a.dv = dv;
  a.kv_v8 = ((reinterpret_cast<uintptr_t>(dk) | reinterpret_cast<uintptr_t>(dv)) & 31u) == 0 ? 1 : 0;
  a.rope = path == kBwdFused ? rope : nullptr;
  a.ds = ds;
  a.ds_tt = (G / kTile) * (G / kTile + 1) / 2;
  a.ds_slots = ds_slots;
  a.kv_q128 = (qtile == 128 && seg == nullptr && hist.tiles == nullptr && path != kBwdFused) ? 1 : 0;
  a.ds_blocks = ds_blocks;
  a.status = status;
  a.wait_limit_ns = wait_limit_ns();
  int launches = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (path == kBwdFused)
    e = launch_bwd_fused<128>(maps, pre, a, info.sms, s, &launches);  // the plan picks it at D == 128 only
  else
    e = (D == 64) ? launch_bwd<64>(maps, pre, a, info.sms, s, &launches, stages)
                  : launch_bwd<128>(maps, pre, a, info.sms, s, &launches, stages);
  if (e == cudaSuccess && rope != nullptr && path != kBwdFused) {
    // the split path writes dq, dk of the rotated inputs: turn them back in place
    e = launch_rope_apply(dq, dq, rope, B, N, H, D, 1, info.sms, s);
    if (e == cudaSuccess) e = launch_rope_apply(dk, dk, rope, B, N, Hkv, D, 1, info.sms, s);
    launches += 2;
  }
  g_last_launches = launches;
  if (e != cudaSuccess) g_last_cuda_error = static_cast<int>(e);
  return e == cudaSuccess ? S2ATTN_OK : S2ATTN_ERR_CUDA;
}

bool rope_table_args_ok(int N, int D, double pos_scale, double base) {
  return N > 0 && (D == 64 || D == 128) && pos_scale > 0.0 && pos_scale <= 1e6 && base > 1.0 && base < 1e30;
}
}  // namespace

extern "C" {

int s2attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
               const void* dO, void* dq, void* dk, void* dv, int B, int H, int Hkv, int N, int D,
               int G, void* workspace, size_t workspace_bytes, s2attn_stream_t stream) {
  const Plan plan = select_plan(B, H, Hkv, N, D, G, 0);
  return bwd_impl(plan.bwd_path, plan.bwd_stages, plan.ds_slots, plan.bwd_qtile, q, k, v, o, lse, dO, dq, dk, dv, B, H, Hkv, N, D, G,
                  workspace, workspace_bytes, stream);
}

size_t s2attn_rope_table_bytes(int N, int D) {
  if (N <= 0 || (D != 64 && D != 128)) return 0;
  return static_cast<size_t>(N) * (D / 2) * 2 * sizeof(float);
}

int s2attn_rope_table(float* table, int N, int D, double pos_scale, double rope_base, s2attn_stream_t stream) {
  g_last_launches = 0;
  if (!table) return S2ATTN_ERR_INVALID_ARG;
  if (!rope_table_args_ok(N, D, pos_scale, rope_base)) return D == 64 || D == 128 ? S2ATTN_ERR_INVALID_ARG
                                                                                 : S2ATTN_ERR_UNSUPPORTED;
  if (!aligned16(table)) return S2ATTN_ERR_MISALIGNED;
  DeviceInfo info;
  if (!device_info(&info)) return S2ATTN_ERR_CUDA;
  if (!info.ok) return S2ATTN_ERR_UNSUPPORTED;
  if (launch_rope_table(table, N, D, pos_scale, rope_base, info.sms, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return S2ATTN_ERR_CUDA;
  g_last_launches = 1;
  return S2ATTN_OK;
}

int s2attn_rope_apply(const void* x, void* out, const float* table, int B, int N, int heads, int D, int inverse,
                      s2attn_stream_t stream) {
  g_last_launches = 0;
  if (!x || !out || !table || B <= 0 || N <= 0 || heads <= 0) return S2ATTN_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return S2ATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * N * heads * D >= (1LL << 40)) return S2ATTN_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(out) || !aligned16(table)) return S2ATTN_ERR_MISALIGNED;
  DeviceInfo info;
  if (!device_info(&info)) return S2ATTN_ERR_CUDA;
  if (!info.ok) return S2ATTN_ERR_UNSUPPORTED;
  if (launch_rope_apply(x, out, table, B, N, heads, D, inverse ? 1 : 0, info.sms,
                        static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return S2ATTN_ERR_CUDA;
  g_last_launches = 1;
  return S2ATTN_OK;
}

int s2attn_fwd_rope(const void* q, const void* k, const void* v, void* o, float* lse, void* q_rot, void* k_rot,
                    const float* table, int B, int H, int Hkv, int N, int D, int G, s2attn_stream_t stream) {
  g_last_launches = 0;
  if (!q || !k || !v || !o || !lse || !q_rot || !k_rot || !table) return S2ATTN_ERR_INVALID_ARG;
  int st = validate_shape(B, H, Hkv, N, D, G);
  if (st != S2ATTN_OK) return st;
  if (!aligned16(q) || !aligned16(k) || !aligned16(q_rot) || !aligned16(k_rot) || !aligned16(table))
    return S2ATTN_ERR_MISALIGNED;
  if (q_rot == q || k_rot == k || q_rot == k_rot) return S2ATTN_ERR_INVALID_ARG;  // the backward needs both
  st = s2attn_rope_apply(q, q_rot, table, B, N, H, D, 0, stream);
  if (st != S2ATTN_OK) return st;
  st = s2attn_rope_apply(k, k_rot, table, B, N, Hkv, D, 0, stream);
  if (st != S2ATTN_OK) return st;
  st = s2attn_fwd(q_rot, k_rot, v, o, lse, B, H, Hkv, N, D, G, stream);
  g_last_launches = st == S2ATTN_OK ? 3 : 0;
  return st;
}

int s2attn_bwd_rope(const void* q_rot, const void* k_rot, const void* v, const void* o, const float* lse,
                    const void* dO, void* dq, void* dk, void* dv, const float* table, int B, int H, int Hkv, int N,
                    int D, int G, void* workspace, size_t workspace_bytes, s2attn_stream_t stream) {
  g_last_launches = 0;
  if (!table) return S2ATTN_ERR_INVALID_ARG;
  if (!aligned16(table)) return S2ATTN_ERR_MISALIGNED;
  const Plan plan = select_plan(B, H, Hkv, N, D, G, 0);
  return bwd_impl(plan.bwd_path, plan.bwd_stages, plan.ds_slots, plan.bwd_qtile, q_rot, k_rot, v, o, lse, dO, dq, dk, dv, B, H, Hkv, N, D, G,
                  workspace, workspace_bytes, stream, table);
}

size_t s2attn_seg_bwd_workspace_bytes(int B, int H, int Hkv, int N, int Nk, int D) {
  if (validate_segment(B, H, Hkv, N, Nk, D, 0) != S2ATTN_OK) return 0;
  return workspace_bytes_for(kBwdSplit, B, H, N, D);
}

int s2attn_seg_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                   void* dq, void* dk, void* dv, int B, int H, int Hkv, int N, int Nk, int D, int causal,
                   int dq_accumulate, void* workspace, size_t workspace_bytes, s2attn_stream_t stream) {
  g_last_launches = 0;
  const int st = validate_segment(B, H, Hkv, N, Nk, D, causal);
  if (st != S2ATTN_OK) return st;
  const Dims d = make_segment_dims(B, H, Hkv, N, Nk, D, causal);
  const Plan plan = select_plan(B, H, Hkv, N, D, N, 0);
  return bwd_impl(kBwdSplit, plan.bwd_stages, 0, 64, q, k, v, o, lse, dO, dq, dk, dv, B, H, Hkv, N, D, N, workspace,
                  workspace_bytes, stream, nullptr, &d, dq_accumulate);
}

int s2attn_lse_merge(const void* o_a, const float* lse_a, const void* o_b, const float* lse_b, void* o, float* lse,
                     int B, int H, int N, int D, s2attn_stream_t stream) {
  g_last_launches = 0;
  if (!o_a || !lse_a || !o_b || !lse_b || !o || !lse || B <= 0 || H <= 0 || N <= 0) return S2ATTN_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return S2ATTN_ERR_UNSUPPORTED;
  if (N % kTile != 0 || static_cast<long long>(B) * N * H * D >= (1LL << 40)) return S2ATTN_ERR_UNSUPPORTED;
  if (!aligned16(o_a) || !aligned16(o_b) || !aligned16(o) || !aligned16(lse_a) || !aligned16(lse_b) ||
      !aligned16(lse))
    return S2ATTN_ERR_MISALIGNED;
  DeviceInfo info;
  if (!device_info(&info)) return S2ATTN_ERR_CUDA;
  if (!info.ok) return S2ATTN_ERR_UNSUPPORTED;
  if (launch_lse_merge(o_a, lse_a, o_b, lse_b, o, lse, B, H, N, D, info.sms, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return S2ATTN_ERR_CUDA;
  g_last_launches = 1;
  return S2ATTN_OK;
}

int s2attn_hga_fwd(const void* q, const void* k, const void* v, void* o, float* lse, const int* hist, int S,
                   int B, int H, int Hkv, int N, int D, int G, s2attn_stream_t stream) {
  g_last_launches = 0;
  if (!q || !k || !v || !o || !lse || (S > 0 && !hist) || S < 0 || S > 4096) return S2ATTN_ERR_INVALID_ARG;
  int st = validate_shape(B, H, Hkv, N, D, G, false);
  if (st != S2ATTN_OK) return st;
  if (G % kQBlock != 0) return S2ATTN_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(hist) & 3u) != 0) return S2ATTN_ERR_MISALIGNED;
  Dims d = make_dims(B, H, Hkv, N, D, G);
  d.noshift = 1;
  HgaList hl;
  hl.tiles = hist;
  hl.S = S;
  return fwd_impl(q, k, v, o, lse, d, stream, hl);
}

int s2attn_hga_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                   void* dq, void* dk, void* dv, const int* hist, int S, int B, int H, int Hkv, int N, int D, int G,
                   void* workspace, size_t workspace_bytes, s2attn_stream_t stream) {
  g_last_launches = 0;
  if ((S > 0 && !hist) || S < 0 || S > 4096) return S2ATTN_ERR_INVALID_ARG;
  int st = validate_shape(B, H, Hkv, N, D, G, false);
  if (st != S2ATTN_OK) return st;
  if (G % kQBlock != 0) return S2ATTN_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(hist) & 3u) != 0) return S2ATTN_ERR_MISALIGNED;
  Dims d = make_dims(B, H, Hkv, N, D, G);
  d.noshift = 1;
  HgaList hl;
  hl.tiles = hist;
  hl.S = S;
  const Plan plan = select_plan(B, H, Hkv, N, D, G, 0);
  return bwd_impl(kBwdSplit, plan.bwd_stages, 0, 64, q, k, v, o, lse, dO, dq, dk, dv, B, H, Hkv, N, D, G, workspace,
                  workspace_bytes, stream, nullptr, &d, 0, hl);
}

}  // extern "C"

namespace {
// ---------------------------------------------------------------- NF4
// Phi^-1(p), the standard normal quantile, by bisection on the normal CDF
// written through erfc (double precision; 200 halvings of [-10, 10]).
double normal_quantile(double p) {
  double lo = -10.0, hi = 10.0;
  for (int i = 0; i < 200; ++i) {
    const double mid = 0.5 * (lo + hi);
    if (0.5 * std::erfc(-mid / std::sqrt(2.0)) < p)
      lo = mid;
    else
      hi = mid;
  }
  return 0.5 * (lo + hi);
}

// The 16 NF4 levels (QLoRA's 4-bit NormalFloat): standard normal quantiles
// normalised into [-1, 1] with an exact zero.  With delta = (1/30 + 1/32) / 2
// and top = Phi^-1(1 - delta): the zero and 8 positive levels are
// Phi^-1(p) / top at 9 evenly spaced p from 1/2 to 1 - delta; the 7 negative
// levels are -Phi^-1(p) / top at 8 such p, the first (the zero) dropped.
// Ascending, so the code is the index.
const Nf4Levels& nf4_levels() {
  static const Nf4Levels lv = [] {
    Nf4Levels t;
    const double delta = 0.5 * (1.0 / 30.0 + 1.0 / 32.0);
    const double top = normal_quantile(1.0 - delta);
    for (int i = 1; i < 8; ++i) t.v[7 - i] = static_cast<float>(-normal_quantile(0.5 + (0.5 - delta) * i / 7.0) / top);
    t.v[7] = 0.f;
    for (int i = 1; i < 9; ++i) t.v[7 + i] = static_cast<float>(normal_quantile(0.5 + (0.5 - delta) * i / 8.0) / top);
    return t;
  }();
  return lv;
}

// Variant of the fused NF4 projection: 5 stages and 8 dequantization warps,
// or the override's nf4_stages=4|5 and nf4_dq=8|12 (12 warps with 5 stages).
int nf4_stages() {
  const std::string v = override_value(tile_override(), "nf4_stages");
  return v == "4" ? 4 : 5;
}
int nf4_dq_warps() {
  const std::string v = override_value(tile_override(), "nf4_dq");
  return v == "12" && nf4_stages() == 5 ? 12 : 8;
}

int validate_nf4(int M, int K, int H, int Hkv, int D) {
  if (M <= 0 || K <= 0 || H <= 0 || Hkv <= 0 || D <= 0) return S2ATTN_ERR_INVALID_ARG;
  if (K % 64 != 0) return S2ATTN_ERR_UNSUPPORTED;
  const long long wq = static_cast<long long>(H) * D, wk = static_cast<long long>(Hkv) * D;
  if (wq % 128 != 0 || wk % 128 != 0) return S2ATTN_ERR_UNSUPPORTED;
  const long long nout = wq + 2 * wk;
  if (nout >= (1LL << 24) || M >= (1 << 30) || K >= (1 << 24)) return S2ATTN_ERR_UNSUPPORTED;
  if (nout * (K / 64) >= (1LL << 31) || static_cast<long long>(M) * K >= (1LL << 40) ||
      static_cast<long long>(M) * nout >= (1LL << 40))
    return S2ATTN_ERR_UNSUPPORTED;
  return S2ATTN_OK;
}
}  // namespace

extern "C" {

int s2attn_nf4_levels(float* levels) {
  if (!levels) return S2ATTN_ERR_INVALID_ARG;
  for (int i = 0; i < 16; ++i) levels[i] = nf4_levels().v[i];
  return S2ATTN_OK;
}

int s2attn_nf4_dequant(const void* codes, const int8_t* scale_codes, const float* c2, void* w, int rows, int K,
                       s2attn_stream_t stream) {
  g_last_launches = 0;
  if (!codes || !scale_codes || !c2 || !w || rows <= 0 || K <= 0) return S2ATTN_ERR_INVALID_ARG;
  if (K % 64 != 0) return S2ATTN_ERR_UNSUPPORTED;
  const long long blocks = static_cast<long long>(rows) * (K / 64);
  if (blocks >= (1LL << 31)) return S2ATTN_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(codes) & 3u) != 0 || (reinterpret_cast<uintptr_t>(c2) & 3u) != 0 ||
      !aligned16(w))
    return S2ATTN_ERR_MISALIGNED;
  DeviceInfo info;
  if (!device_info(&info)) return S2ATTN_ERR_CUDA;
  if (!info.ok) return S2ATTN_ERR_UNSUPPORTED;
  const cudaError_t e = launch_nf4_dequant(codes, scale_codes, c2, w, blocks * 8, nf4_levels(), info.sms,
                                           static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    g_last_cuda_error = static_cast<int>(e);
    return S2ATTN_ERR_CUDA;
  }
  g_last_launches = 1;
  return S2ATTN_OK;
}

int s2attn_nf4_qkv(const void* x, const void* codes, const int8_t* scale_codes, const float* c2, void* q, void* k,
                   void* v, int M, int K, int H, int Hkv, int D, s2attn_stream_t stream) {
  g_last_launches = 0;
  if (!x || !codes || !scale_codes || !c2 || !q || !k || !v) return S2ATTN_ERR_INVALID_ARG;
  const int st = validate_nf4(M, K, H, Hkv, D);
  if (st != S2ATTN_OK) return st;
  if (!aligned16(x) || !aligned16(codes) || (reinterpret_cast<uintptr_t>(c2) & 3u) != 0 || !aligned16(q) ||
      !aligned16(k) || !aligned16(v))
    return S2ATTN_ERR_MISALIGNED;
  DeviceInfo info;
  if (!device_info(&info)) return S2ATTN_ERR_CUDA;
  if (!info.ok) return S2ATTN_ERR_UNSUPPORTED;
  const int nout = (H + 2 * Hkv) * D;
  CUtensorMap tx, tc;
  if (!make_map_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, static_cast<uint64_t>(K), static_cast<uint64_t>(M),
                   static_cast<uint64_t>(K) * 2, 64, 256, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&tc, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, static_cast<uint64_t>(K / 2),
                   static_cast<uint64_t>(nout), static_cast<uint64_t>(K / 2), 32, 128, CU_TENSOR_MAP_SWIZZLE_NONE))
    return S2ATTN_ERR_CUDA;
  CUtensorMap to[3];
  const void* outs[3] = {q, k, v};
  const int widths[3] = {H * D, Hkv * D, Hkv * D};
  for (int i = 0; i < 3; ++i)
    if (!make_map_2d(&to[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, outs[i], static_cast<uint64_t>(widths[i]),
                     static_cast<uint64_t>(M), static_cast<uint64_t>(widths[i]) * 2, 32, 128,
                     CU_TENSOR_MAP_SWIZZLE_NONE))
      return S2ATTN_ERR_CUDA;
  Nf4Args a;
  a.sq = scale_codes;
  a.c2 = c2;
  a.width0 = H * D;
  a.width1 = Hkv * D;
  a.M = M;
  a.K = K;
  a.tiles_w = nout / 128;
  a.tiles_t = (M + 255) / 256;
  a.lv = nf4_levels();
  void* status = nullptr;
  const cudaError_t se = cudaGetSymbolAddress(&status, g_fwd_status);
  if (se != cudaSuccess) {
    g_last_cuda_error = static_cast<int>(se);
    return S2ATTN_ERR_CUDA;
  }
  a.status = static_cast<uint32_t*>(status);
  a.wait_limit_ns = wait_limit_ns();
  const cudaError_t e = launch_nf4_qkv(tx, tc, to, a, info.sms, static_cast<cudaStream_t>(stream), nf4_stages(),
                                       nf4_dq_warps());
  if (e != cudaSuccess) {
    g_last_cuda_error = static_cast<int>(e);
    return S2ATTN_ERR_CUDA;
  }
  g_last_launches = 1;
  return S2ATTN_OK;
}

size_t s2attn_hga_bwd_workspace_bytes(int B, int H, int Hkv, int N, int D, int G) {
  if (validate_shape(B, H, Hkv, N, D, G, false) != S2ATTN_OK || G % kQBlock != 0) return 0;
  return workspace_bytes_for(kBwdSplit, B, H, N, D);
}

int s2attn_plan(int B, int H, int Hkv, int N, int D, int G, int num_sms, int* out) {
  if (!out) return S2ATTN_ERR_INVALID_ARG;
  const int st = validate_shape(B, H, Hkv, N, D, G);
  if (st != S2ATTN_OK) return st;
  const Plan p = select_plan(B, H, Hkv, N, D, G, num_sms);
  out[0] = p.fwd_snake;
  out[1] = p.fwd_kv_slots;
  out[2] = p.bwd_path;
  out[3] = p.bwd_stages;
  out[4] = p.fwd_bn;
  out[5] = p.bwd_path == kBwdSplitDs ? p.ds_slots : 0;
  out[6] = p.bwd_qtile;
  return S2ATTN_OK;
}

int s2attn_set_tile_override(const char* spec) {
  std::lock_guard<std::mutex> lk(g_override_mu);
  if (spec) {
    g_override = spec;
  } else {
    const char* e = std::getenv("S2ATTN_TILE");
    g_override = e ? e : "";
  }
  g_override_init = true;
  return S2ATTN_OK;
}


int s2attn_device_status(void* workspace, s2attn_stream_t stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return S2ATTN_ERR_CUDA;
  uint32_t words[2] = {0, 0};
  const uint32_t zero[2] = {0, 0};
  if (workspace) {
    if (cudaMemcpy(words, workspace, sizeof(words), cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemcpy(workspace, zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
      return S2ATTN_ERR_CUDA;
  } else {
    if (cudaMemcpyFromSymbol(words, g_fwd_status, sizeof(words)) != cudaSuccess ||
        cudaMemcpyToSymbol(g_fwd_status, zero, sizeof(zero)) != cudaSuccess)
      return S2ATTN_ERR_CUDA;
  }
  return words[0] == 0 ? S2ATTN_OK : static_cast<int>(words[0]);
}

int s2attn_selftest_wait_timeout(uint32_t* status_out, uint64_t limit_ns, s2attn_stream_t stream) {
  if (!status_out || limit_ns == 0 || limit_ns > 10000000000ull) return S2ATTN_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(status_out) & 7u) != 0) return S2ATTN_ERR_MISALIGNED;
  DeviceInfo info;
  if (!device_info(&info)) return S2ATTN_ERR_CUDA;
  if (!info.ok) return S2ATTN_ERR_UNSUPPORTED;
  s2_selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(status_out, limit_ns);
  return cudaGetLastError() == cudaSuccess ? S2ATTN_OK : S2ATTN_ERR_CUDA;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Backward for callers that cannot allocate device memory.
//
// Some callers have no way to obtain device memory for a workspace: code that
// runs under another runtime's memory budget with no allocator handle, plugin
// hosts that forbid cudaMalloc, or programs that must not allocate between
// set-up and capture.  For them the backward's scratch (status block, Delta and
// lse*log2(e), s2attn_bwd_workspace_bytes of it) lives in this fixed array.
// Every GPU that loads the library reserves it when the module is loaded and
// keeps it until the process exits.  All calls share it and it keeps the last
// call's contents; the backward's first kernel rewrites everything the later
// kernels read (and clears the status words), so nothing needs clearing here.
// Calls that overlap on the GPU (different streams, or devices sharing a
// context) race on the array.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_bwd_scratch[kNoAllocScratchBytes];

// Device address of g_bwd_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up with
// the device current, once per device and context, and cached.  The cache is
// keyed on the current context as well as the device index: a context torn
// down and recreated (cudaDeviceReset) loads the module again at a new
// address, so a changed context handle triggers a new lookup.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

CtxGetCurrentFn get_ctx_current() {
  static std::once_flag once;
  static CtxGetCurrentFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

bool noalloc_scratch(void** out) {
  static std::mutex mu;
  static void* ptrs[64] = {};
  static CUcontext ctxs[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  CtxGetCurrentFn ctx_current = get_ctx_current();
  if (!ctx_current) return false;
  std::lock_guard<std::mutex> lk(mu);
  CUcontext ctx = nullptr;
  // the runtime makes the device's primary context current on first use;
  // before that there is none and the lookup below creates it
  if (ctx_current(&ctx) != CUDA_SUCCESS) return false;
  if (ptrs[dev] == nullptr || ctx == nullptr || ctx != ctxs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_bwd_scratch) != cudaSuccess || p == nullptr) return false;
    if (ctx_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
    ptrs[dev] = p;
    ctxs[dev] = ctx;
  }
  *out = ptrs[dev];
  return true;
}

}  // namespace

extern "C" int s2attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                  const float* lse, const void* dO, void* dq, void* dk, void* dv,
                                  int B, int H, int Hkv, int N, int D, int G,
                                  s2attn_stream_t stream) {
  g_last_launches = 0;
  // the split backward: its scratch (status block, Delta, lse*log2(e)) grows
  // with B * H * N only, where the fused path would need a dQ accumulator of
  // B * H * N * D floats
  const bool valid = validate_shape(B, H, Hkv, N, D, G) == S2ATTN_OK;
  const size_t need = valid ? workspace_bytes_for(kBwdSplit, B, H, N, D) : 0;
  if (need > kNoAllocScratchBytes) return S2ATTN_ERR_WORKSPACE;
  void* scratch = nullptr;
  // an invalid shape: bwd_impl reports which error
  if (valid && !noalloc_scratch(&scratch)) return S2ATTN_ERR_CUDA;
  const Plan plan = select_plan(B, H, Hkv, N, D, G, 0);
  return bwd_impl(kBwdSplit, plan.bwd_stages, 0, plan.bwd_qtile, q, k, v, o, lse, dO, dq, dk, dv, B, H, Hkv, N, D, G, scratch,
                  kNoAllocScratchBytes, stream);
}
