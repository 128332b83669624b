// C ABI of libslim.so (declared in include/slim.h): argument checks,
// workspace carve-up, kernel selection and the measured ordering table.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "slim_internal.h"

namespace slim {

// ---------------------------------------------------------------------------- device queries
int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return 148;  // B200
  }
  return n;
}

int max_smem_optin() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return 232448;  // B200: 227 KiB
  }
  return n;
}

// ---------------------------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

bool encode_tmap_2d_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                         uint32_t box_inner, uint32_t box_outer, bool swizzle128) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_tmap_3d_bf16(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1,
                         uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1, s2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_tmap(CUtensorMap* map, CUtensorMapDataType type, int rank, const void* base, const uint64_t* dims,
                 const uint64_t* strides, const uint32_t* box, bool swizzle128) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn || rank < 1 || rank > 5) return false;
  cuuint64_t dd[5], ss[4];
  cuuint32_t bb[5], ee[5];
  for (int i = 0; i < rank; ++i) {
    dd[i] = dims[i];
    bb[i] = box[i];
    ee[i] = 1;
    if (i + 1 < rank) ss[i] = strides[i];
  }
  CUresult r = fn(map, type, static_cast<cuuint32_t>(rank), const_cast<void*>(base), dd, ss, bb, ee,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_tmap_kslab(CUtensorMap* map, const void* base, uint64_t rows, int d, int box_blocks) {
  if (d % 64 || box_blocks < 1 || box_blocks > 256) return false;
  return encode_tmap_3d_bf16(map, base, 64, rows, static_cast<uint64_t>(d / 64), static_cast<uint64_t>(d) * 2u, 128,
                             64, 16, static_cast<uint32_t>(box_blocks));
}

// ---------------------------------------------------------------------------- workspace
namespace {

constexpr size_t kAlign = 256;
size_t up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }
size_t esize(int dtype) { return dtype == SLIM_BF16 ? 2 : 4; }

struct WsLayout {
  size_t U, m, l, meta, vbuf, stage, total;
  int max_items;
};

WsLayout ws_layout(int dtype, int B, int d, int H, int64_t cap, int variant) {
  WsLayout w{};
  // partial slots: a split kernel runs at most num_sms() work groups, and a group's contiguous share
  // of the rows adds one slot per sequence boundary inside it
  const int items = num_sms() + B;
  w.max_items = items;
  const bool need_b = variant != SLIM_VARIANT_A;
  const bool need_a = variant != SLIM_VARIANT_B;
  // ordering (a) on tensor cores keeps V in TMEM: one partial of 256 columns (4 heads' m, l) per tile
  const bool a_tc = need_a && decode_a_tc_supported(dtype, B, d, H);
  const size_t a_tiles = a_tc ? decode_a_tc_slots(B, d, cap) : 0;
  size_t u_floats = 0, ml_floats = static_cast<size_t>(items) * H;
  if (need_b) u_floats = std::max(u_floats, static_cast<size_t>(items) * H * d);
  if (need_a && !a_tc) u_floats = std::max(u_floats, static_cast<size_t>(items) * d);
  if (a_tc) {
    u_floats = std::max(u_floats, a_tiles * 256);
    ml_floats = std::max(ml_floats, a_tiles * 4);
  }
  size_t o = 0;
  w.U = o;
  o += up(u_floats * 4);
  w.m = o;
  o += up(ml_floats * 4);
  w.l = o;
  o += up(ml_floats * 4);
  w.meta = o;
  o += up(meta_ints(B) * 4);
  w.vbuf = o;
  if (need_a && !a_tc) o += up(static_cast<size_t>(B) * cap * d * esize(dtype));
  w.stage = o;
  o += up(static_cast<size_t>(B) * d * 4) * 2 + up(static_cast<size_t>(B) * d * esize(dtype));
  w.total = o;
  return w;
}

SplitWorkspace carve(void* base, const WsLayout& w) {
  char* c = static_cast<char*>(base);
  SplitWorkspace s;
  s.U = reinterpret_cast<float*>(c + w.U);
  s.m = reinterpret_cast<float*>(c + w.m);
  s.l = reinterpret_cast<float*>(c + w.l);
  s.meta = reinterpret_cast<int32_t*>(c + w.meta);
  s.vbuf = c + w.vbuf;
  s.qstage = c + w.stage;
  s.max_items = w.max_items;
  return s;
}

thread_local int g_last_launches = 0;

// Test hook of the failure path (slim_debug_stall_next): armed for one call on this thread.
struct StallHook {
  uint64_t wait_ns = 0;
  bool armed = false;
};
thread_local StallHook g_stall;

// Measurement aid: event pairs recorded around the split kernel.
struct TimingRing {
  std::vector<cudaEvent_t> start, stop;
  int next = 0, recorded = 0;
};
thread_local TimingRing g_timing;

void timing_before(cudaStream_t st) {
  if (g_timing.start.empty()) return;
  cudaEventRecord(g_timing.start[g_timing.next], st);
}
void timing_after(cudaStream_t st) {
  if (g_timing.start.empty()) return;
  cudaEventRecord(g_timing.stop[g_timing.next], st);
  g_timing.next = (g_timing.next + 1) % static_cast<int>(g_timing.start.size());
  g_timing.recorded = std::min(g_timing.recorded + 1, static_cast<int>(g_timing.start.size()));
}

// ---------------------------------------------------------------------------- ordering table
struct TuneKey {
  int dtype, B, d, H;
  bool operator<(const TuneKey& o) const {
    return std::tie(dtype, B, d, H) < std::tie(o.dtype, o.B, o.d, o.H);
  }
};
struct TunePoint {
  int64_t T;
  float ms_a, ms_b;
};
std::mutex g_tune_mu;
std::map<TuneKey, std::vector<TunePoint>> g_tune;

bool valid_dims(int dtype, int B, int d, int H, int64_t cap) {
  return (dtype == SLIM_F32 || dtype == SLIM_BF16) && B >= 1 && d >= 1 && H >= 1 && d % H == 0 && cap >= 1 &&
         cap <= (int64_t(1) << 31) - 1 && static_cast<int64_t>(B) * cap <= (int64_t(1) << 31) - 1;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

cudaError_t launch_prefill_simt(const void* X, const void* W, void* kcache, const int32_t* lens, int dtype, int B,
                                int n, int d, int64_t cap, cudaStream_t st, int* launches);
cudaError_t launch_prefill_tc(const void* X, const void* W, void* kcache, const int32_t* lens, int B, int n, int d,
                              int64_t cap, int32_t* status, cudaStream_t st, int* launches);
bool gemm_tc_supported(int d);
cudaError_t launch_advance_lens(int32_t* lens, int B, int n, int64_t cap, int32_t* status, cudaStream_t st,
                                int* launches);

cudaError_t launch_rows_gemm_any(const void* A, const void* W, void* Y, const int32_t* lens, int rows_extra,
                                 int dtype, int B, int d, int64_t cap, int32_t* status, cudaStream_t st,
                                 int* launches) {
  if (dtype == SLIM_BF16 && gemm_tc_supported(d))
    return launch_rows_gemm_tc(A, W, Y, lens, rows_extra, B, d, cap, status, st, launches);
  return launch_rows_gemm(A, W, Y, lens, rows_extra, dtype, B, d, cap, st, launches);
}

}  // namespace slim

using namespace slim;

// ============================================================================ C ABI
extern "C" {

int slim_version(void) { return 100; }

int slim_timing_enable(int n) {
  if (n < 0) return SLIM_EINVAL;
  for (auto e : g_timing.start) cudaEventDestroy(e);
  for (auto e : g_timing.stop) cudaEventDestroy(e);
  g_timing = TimingRing{};
  for (int i = 0; i < n; ++i) {
    cudaEvent_t a, b;
    if (cudaEventCreate(&a) != cudaSuccess || cudaEventCreate(&b) != cudaSuccess) {
      cudaGetLastError();
      return SLIM_ECUDA;
    }
    g_timing.start.push_back(a);
    g_timing.stop.push_back(b);
  }
  return SLIM_OK;
}

int slim_timing_read(float* ms, int n) {
  if (!ms || n < 0) return SLIM_EINVAL;
  const int cnt = std::min(n, g_timing.recorded);
  for (int i = 0; i < cnt; ++i) {
    if (cudaEventElapsedTime(&ms[i], g_timing.start[i], g_timing.stop[i]) != cudaSuccess) {
      cudaGetLastError();
      return SLIM_ECUDA;
    }
  }
  return cnt;
}

int slim_last_launch_count(void) { return g_last_launches; }

int slim_debug_stall_next(int64_t wait_ns) {
  if (wait_ns < 1000 || wait_ns > static_cast<int64_t>(kWaitLimitNs)) return SLIM_EINVAL;
  g_stall.wait_ns = static_cast<uint64_t>(wait_ns);
  g_stall.armed = true;
  return SLIM_OK;
}

const char* slim_strerror(int code) {
  switch (code) {
    case SLIM_OK: return "success";
    case SLIM_EINVAL: return "invalid argument (null pointer, size, d % H, dtype or variant)";
    case SLIM_EWORKSPACE: return "workspace missing, too small or not 256-byte aligned";
    case SLIM_ECUDA: return "CUDA runtime or launch failure";
    case SLIM_EUNSUPPORTED: return "no kernel for this shape/dtype";
    case SLIM_DEV_OVERFLOW: return "device: append would exceed cache capacity (sequence skipped)";
    case SLIM_DEV_BADLEN: return "device: length outside [0, cap] (sequence skipped)";
    case SLIM_DEV_TIMEOUT: return "device: a bounded wait gave up (internal error)";
    default: break;
  }
  if (code > 0 && code < 8) return "device: several status bits set";
  return "unknown code";
}

int slim_prefill_k(const void* X, const void* W_K, void* Kcache, int32_t* lens, int dtype, int B, int n, int d,
                   int64_t cap, int32_t* dev_status, void* stream) {
  if (!X || !W_K || !Kcache || !lens || !dev_status || n < 1) return SLIM_EINVAL;
  if (!valid_dims(dtype, B, d, 1, cap)) return SLIM_EINVAL;
  if (static_cast<int64_t>(n) > cap) return SLIM_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int launches = 0;
  cudaError_t e;
  if (dtype == SLIM_BF16 && gemm_tc_supported(d) && aligned(X, 16) && aligned(W_K, 16) && aligned(Kcache, 16))
    e = launch_prefill_tc(X, W_K, Kcache, lens, B, n, d, cap, dev_status, st, &launches);
  else
    e = launch_prefill_simt(X, W_K, Kcache, lens, dtype, B, n, d, cap, st, &launches);
  if (e == cudaSuccess) e = launch_advance_lens(lens, B, n, cap, dev_status, st, &launches);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return e == cudaErrorNotSupported ? SLIM_EUNSUPPORTED : SLIM_ECUDA;
  }
  g_last_launches = launches;
  return SLIM_OK;
}

size_t slim_decode_workspace_bytes(int dtype, int B, int d, int H, int64_t cap, int variant) {
  if (!valid_dims(dtype, B, d, H, cap) || variant < SLIM_AUTO || variant > SLIM_VARIANT_B) return 0;
  return ws_layout(dtype, B, d, H, cap, variant).total;
}

int slim_select_variant(int dtype, int B, int d, int H, int64_t T) {
  std::lock_guard<std::mutex> g(g_tune_mu);
  auto it = g_tune.find(TuneKey{dtype, B, d, H});
  if (it == g_tune.end() || it->second.empty() || T < 1) return SLIM_VARIANT_B;
  const TunePoint* best = nullptr;
  double bestd = 0;
  for (const auto& p : it->second) {
    const double dist = std::fabs(std::log(static_cast<double>(p.T)) - std::log(static_cast<double>(T)));
    if (!best || dist < bestd) {
      best = &p;
      bestd = dist;
    }
  }
  return (best->ms_a < best->ms_b) ? SLIM_VARIANT_A : SLIM_VARIANT_B;
}

int slim_tune_record(int dtype, int B, int d, int H, int64_t T, float ms_a, float ms_b) {
  if (!valid_dims(dtype, B, d, H, T) || !(ms_a > 0.f) || !(ms_b > 0.f)) return SLIM_EINVAL;
  std::lock_guard<std::mutex> g(g_tune_mu);
  auto& v = g_tune[TuneKey{dtype, B, d, H}];
  for (auto& p : v)
    if (p.T == T) {
      p.ms_a = ms_a;
      p.ms_b = ms_b;
      return SLIM_OK;
    }
  v.push_back(TunePoint{T, ms_a, ms_b});
  return SLIM_OK;
}

void slim_tune_clear(void) {
  std::lock_guard<std::mutex> g(g_tune_mu);
  g_tune.clear();
}

int slim_decode_step(const float* q, const void* k_new, void* Kcache, int32_t* lens, const void* W_KV, int dtype,
                     int B, int d, int H, int64_t cap, int variant, int64_t t_hint, float* out, void* workspace,
                     size_t ws_bytes, int32_t* dev_status, void* stream) {
  if (!q || !Kcache || !lens || !W_KV || !out || !dev_status) return SLIM_EINVAL;
  if (!valid_dims(dtype, B, d, H, cap) || variant < SLIM_AUTO || variant > SLIM_VARIANT_B) return SLIM_EINVAL;
  if (!aligned(q, 16) || !aligned(Kcache, 16) || (k_new && !aligned(k_new, 16)) || !aligned(W_KV, 16))
    return SLIM_EINVAL;
  if ((static_cast<size_t>(d) * esize(dtype)) % 16 != 0) return SLIM_EUNSUPPORTED;
  if (!workspace || !aligned(workspace, kAlign)) return SLIM_EWORKSPACE;
  const WsLayout wl = ws_layout(dtype, B, d, H, cap, variant);
  if (ws_bytes < wl.total) return SLIM_EWORKSPACE;
  int v = variant;
  if (v == SLIM_AUTO) v = slim_select_variant(dtype, B, d, H, t_hint > 0 ? t_hint : cap);

  DecodeArgs a{q, k_new, Kcache, lens, W_KV, dtype, B, d, H, cap, out, dev_status};
  if (g_stall.armed && v == SLIM_VARIANT_B) {
    a.wait_ns = g_stall.wait_ns;
    a.stall = 1;
    g_stall.armed = false;
  }
  SplitWorkspace ws = carve(workspace, wl);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int launches = 0;
  cudaError_t e = cudaSuccess;
  if (v == SLIM_VARIANT_B) {
    const bool tc = dtype == SLIM_BF16 && decode_b_tc_supported(B, d, H);
    if (!tc && !decode_b_simt_supported(B, d, H)) return SLIM_EUNSUPPORTED;
    timing_before(st);
    e = tc ? launch_decode_b_tc(a, ws, st, &launches) : launch_decode_b_simt(a, ws, st, &launches);
    timing_after(st);
    if (e == cudaSuccess) e = launch_reduce_b(a, ws, /*pdl=*/g_timing.start.empty(), st, &launches);
  } else {
    if (!decode_a_supported(dtype, B, d, H)) return SLIM_EUNSUPPORTED;
    e = launch_decode_a(a, ws, st, &launches);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return e == cudaErrorNotSupported ? SLIM_EUNSUPPORTED : SLIM_ECUDA;
  }
  g_last_launches = launches;
  return SLIM_OK;
}

int slim_project_qk(const void* x, const void* W_Q, const void* W_K, int dtype, int B, int d, float* q_out,
                    void* k_out, int32_t* dev_status, void* stream) {
  if (!x || !W_Q || !q_out || !dev_status || (!W_K != !k_out)) return SLIM_EINVAL;
  if (!valid_dims(dtype, B, d, 1, 1)) return SLIM_EINVAL;
  if (!aligned(x, 16) || !aligned(W_Q, 16) || (W_K && !aligned(W_K, 16)) || !aligned(q_out, 16) ||
      (k_out && !aligned(k_out, 16)))
    return SLIM_EINVAL;
  if ((static_cast<size_t>(d) * esize(dtype)) % 16 != 0) return SLIM_EUNSUPPORTED;
  int launches = 0;
  const cudaError_t e = launch_front(x, W_Q, W_K, q_out, k_out, dtype, B, d, dev_status,
                                     static_cast<cudaStream_t>(stream), &launches);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return SLIM_ECUDA;
  }
  g_last_launches = launches;
  return SLIM_OK;
}

size_t slim_decode_step_x_workspace_bytes(int dtype, int B, int d, int H, int64_t cap, int variant) {
  const size_t step = slim_decode_workspace_bytes(dtype, B, d, H, cap, variant);
  if (step == 0) return 0;
  return step + up(static_cast<size_t>(B) * d * 4) + up(static_cast<size_t>(B) * d * esize(dtype));
}

int slim_decode_step_x(const void* x, const void* W_Q, const void* W_K, void* Kcache, int32_t* lens,
                       const void* W_KV, int dtype, int B, int d, int H, int64_t cap, int variant, int64_t t_hint,
                       float* out, void* workspace, size_t ws_bytes, int32_t* dev_status, void* stream) {
  // the step's own checks first, so that a rejected call launches nothing
  if (!x || !W_Q || !Kcache || !lens || !W_KV || !out || !dev_status) return SLIM_EINVAL;
  if (!valid_dims(dtype, B, d, H, cap) || variant < SLIM_AUTO || variant > SLIM_VARIANT_B) return SLIM_EINVAL;
  if (!aligned(x, 16) || !aligned(W_Q, 16) || (W_K && !aligned(W_K, 16)) || !aligned(Kcache, 16) ||
      !aligned(W_KV, 16))
    return SLIM_EINVAL;
  if ((static_cast<size_t>(d) * esize(dtype)) % 16 != 0) return SLIM_EUNSUPPORTED;
  if (!workspace || !aligned(workspace, kAlign)) return SLIM_EWORKSPACE;
  const size_t step = ws_layout(dtype, B, d, H, cap, variant).total;
  if (ws_bytes < slim_decode_step_x_workspace_bytes(dtype, B, d, H, cap, variant)) return SLIM_EWORKSPACE;
  char* w = static_cast<char*>(workspace);
  float* q = reinterpret_cast<float*>(w + step);
  void* k = W_K ? w + step + up(static_cast<size_t>(B) * d * 4) : nullptr;
  int r = slim_project_qk(x, W_Q, W_K, dtype, B, d, q, k, dev_status, stream);
  if (r != SLIM_OK) return r;
  const int front_launches = g_last_launches;
  r = slim_decode_step(q, k, Kcache, lens, W_KV, dtype, B, d, H, cap, variant, t_hint, out, workspace, step,
                       dev_status, stream);
  if (r == SLIM_OK) g_last_launches += front_launches;
  return r;
}

size_t slim_prefill_attention_workspace_bytes(int dtype, int B, int d, int H, int64_t cap) {
  if (!valid_dims(dtype, B, d, H, cap) || !prefill_attn_supported(dtype, d, H)) return 0;
  return up(static_cast<size_t>(B) * cap * d * esize(dtype));  // V = K·W_KV for the cached rows
}

int slim_prefill_attention(const void* Q, const void* Kcache, const int32_t* lens, const void* W_KV, int dtype,
                           int B, int n, int d, int H, int64_t cap, float* out, void* workspace, size_t ws_bytes,
                           int32_t* dev_status, void* stream) {
  if (!Q || !Kcache || !lens || !W_KV || !out || !dev_status || n < 1) return SLIM_EINVAL;
  if (!valid_dims(dtype, B, d, H, cap) || static_cast<int64_t>(n) > cap) return SLIM_EINVAL;
  if (static_cast<int64_t>(B) * n > (int64_t(1) << 31) - 1) return SLIM_EINVAL;
  if (!aligned(Q, 16) || !aligned(Kcache, 16) || !aligned(W_KV, 16) || !aligned(out, 16)) return SLIM_EINVAL;
  if (!prefill_attn_supported(dtype, d, H)) return SLIM_EUNSUPPORTED;
  const size_t need = slim_prefill_attention_workspace_bytes(dtype, B, d, H, cap);
  if (!workspace || !aligned(workspace, kAlign) || ws_bytes < need) return SLIM_EWORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int launches = 0;
  // V = K·W_KV for rows 0 .. lens[b]-1 of every sequence, once for all n queries
  cudaError_t e = launch_rows_gemm_tc(Kcache, W_KV, workspace, lens, 0, B, d, cap, dev_status, st, &launches);
  if (e == cudaSuccess)
    e = launch_prefill_attn(Q, Kcache, workspace, lens, B, n, d, H, cap, out, dev_status, st, &launches);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return e == cudaErrorNotSupported ? SLIM_EUNSUPPORTED : SLIM_ECUDA;
  }
  g_last_launches = launches;
  return SLIM_OK;
}

size_t slim_mha_decode_workspace_bytes(int dtype, int B, int d, int H, int64_t cap) {
  if (!valid_dims(dtype, B, d, H, cap) || dtype != SLIM_BF16 || !decode_kv_supported(B, d, H, cap)) return 0;
  const size_t slots = kv_ws_slots(B, d);
  const int hg = d / 256;
  return up(slots * 256 * 4) + 2 * up(slots * 4 * 4) + up(meta_ints(B * hg) * 4);
}

int slim_mha_decode_step(const float* q, const void* k_new, const void* v_new, void* Kcache, void* Vcache,
                         int32_t* lens, int dtype, int B, int d, int H, int64_t cap, float* out, void* workspace,
                         size_t ws_bytes, int32_t* dev_status, void* stream) {
  if (!q || !Kcache || !Vcache || !lens || !out || !dev_status || (!k_new != !v_new)) return SLIM_EINVAL;
  if (!valid_dims(dtype, B, d, H, cap)) return SLIM_EINVAL;
  if (!aligned(q, 16) || !aligned(Kcache, 16) || !aligned(Vcache, 16) || (k_new && !aligned(k_new, 16)) ||
      (v_new && !aligned(v_new, 16)))
    return SLIM_EINVAL;
  if (dtype != SLIM_BF16 || !decode_kv_supported(B, d, H, cap)) return SLIM_EUNSUPPORTED;
  const size_t need = slim_mha_decode_workspace_bytes(dtype, B, d, H, cap);
  if (!workspace || !aligned(workspace, kAlign) || ws_bytes < need) return SLIM_EWORKSPACE;
  const size_t slots = kv_ws_slots(B, d);
  char* w = static_cast<char*>(workspace);
  float* wsO = reinterpret_cast<float*>(w);
  float* wsm = reinterpret_cast<float*>(w + up(slots * 256 * 4));
  float* wsl = reinterpret_cast<float*>(w + up(slots * 256 * 4) + up(slots * 4 * 4));
  int32_t* meta = reinterpret_cast<int32_t*>(w + up(slots * 256 * 4) + 2 * up(slots * 4 * 4));
  int launches = 0;
  const cudaError_t e = launch_decode_kv(q, k_new, v_new, Kcache, Vcache, lens, B, d, H, cap, out, wsO, wsm, wsl,
                                         meta, dev_status, static_cast<cudaStream_t>(stream), &launches);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return e == cudaErrorNotSupported ? SLIM_EUNSUPPORTED : SLIM_ECUDA;
  }
  g_last_launches = launches;
  return SLIM_OK;
}

int slim_decode_step_host(const float* q_host, const void* k_new_host, void* Kcache, int32_t* lens,
                          const void* W_KV, int dtype, int B, int d, int H, int64_t cap, int variant, int64_t t_hint,
                          float* out_host, void* workspace, size_t ws_bytes, int32_t* dev_status, void* stream) {
  // every check slim_decode_step makes on its own arguments comes first, so that a rejected call
  // has enqueued no copy
  if (!q_host || !out_host || !Kcache || !lens || !W_KV || !dev_status) return SLIM_EINVAL;
  if (!valid_dims(dtype, B, d, H, cap) || variant < SLIM_AUTO || variant > SLIM_VARIANT_B) return SLIM_EINVAL;
  if (!aligned(Kcache, 16) || !aligned(W_KV, 16)) return SLIM_EINVAL;
  if ((static_cast<size_t>(d) * esize(dtype)) % 16 != 0) return SLIM_EUNSUPPORTED;
  if (!workspace || !aligned(workspace, kAlign)) return SLIM_EWORKSPACE;
  const WsLayout wl = ws_layout(dtype, B, d, H, cap, variant);
  if (ws_bytes < wl.total) return SLIM_EWORKSPACE;
  char* stage = static_cast<char*>(workspace) + wl.stage;
  const size_t qb = static_cast<size_t>(B) * d * 4, kb = static_cast<size_t>(B) * d * esize(dtype);
  float* q_dev = reinterpret_cast<float*>(stage);
  float* out_dev = reinterpret_cast<float*>(stage + up(qb));
  void* k_dev = stage + 2 * up(qb);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(q_dev, q_host, qb, cudaMemcpyHostToDevice, st) != cudaSuccess) {
    cudaGetLastError();
    return SLIM_ECUDA;
  }
  if (k_new_host && cudaMemcpyAsync(k_dev, k_new_host, kb, cudaMemcpyHostToDevice, st) != cudaSuccess) {
    cudaGetLastError();
    return SLIM_ECUDA;
  }
  const int r = slim_decode_step(q_dev, k_new_host ? k_dev : nullptr, Kcache, lens, W_KV, dtype, B, d, H, cap,
                                 variant, t_hint, out_dev, workspace, ws_bytes, dev_status, stream);
  if (r != SLIM_OK) return r;
  if (cudaMemcpyAsync(out_host, out_dev, qb, cudaMemcpyDeviceToHost, st) != cudaSuccess) {
    cudaGetLastError();
    return SLIM_ECUDA;
  }
  return SLIM_OK;
}

int slim_tune(const float* q, void* Kcache, int32_t* lens, const int32_t* lens_restore_host, const void* W_KV,
              int dtype, int B, int d, int H, int64_t cap, const int64_t* Ts, int nT, int reps, float* out,
              void* workspace, size_t ws_bytes, int32_t* dev_status, void* stream) {
  if (!Ts || nT < 1 || reps < 1 || !lens_restore_host) return SLIM_EINVAL;
  if (!valid_dims(dtype, B, d, H, cap)) return SLIM_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  std::vector<int32_t> lv(static_cast<size_t>(B));
  cudaEvent_t e0, e1;
  if (cudaEventCreate(&e0) != cudaSuccess || cudaEventCreate(&e1) != cudaSuccess) return SLIM_ECUDA;
  int rc = SLIM_OK;
  for (int i = 0; i < nT && rc == SLIM_OK; ++i) {
    if (Ts[i] < 1 || Ts[i] > cap) {
      rc = SLIM_EINVAL;
      break;
    }
    std::fill(lv.begin(), lv.end(), static_cast<int32_t>(Ts[i]));
    if (cudaMemcpyAsync(lens, lv.data(), lv.size() * 4, cudaMemcpyHostToDevice, st) != cudaSuccess) {
      rc = SLIM_ECUDA;
      break;
    }
    float ms[2] = {0.f, 0.f};
    const int vars[2] = {SLIM_VARIANT_A, SLIM_VARIANT_B};
    for (int k = 0; k < 2 && rc == SLIM_OK; ++k) {
      rc = slim_decode_step(q, nullptr, Kcache, lens, W_KV, dtype, B, d, H, cap, vars[k], 0, out, workspace,
                            ws_bytes, dev_status, stream);  // warm-up
      if (rc != SLIM_OK) break;
      cudaEventRecord(e0, st);
      for (int r = 0; r < reps && rc == SLIM_OK; ++r)
        rc = slim_decode_step(q, nullptr, Kcache, lens, W_KV, dtype, B, d, H, cap, vars[k], 0, out, workspace,
                              ws_bytes, dev_status, stream);
      cudaEventRecord(e1, st);
      if (cudaEventSynchronize(e1) != cudaSuccess) rc = SLIM_ECUDA;
      cudaEventElapsedTime(&ms[k], e0, e1);
      ms[k] /= reps;
    }
    if (rc == SLIM_OK) slim_tune_record(dtype, B, d, H, Ts[i], ms[0], ms[1]);
  }
  if (cudaMemcpyAsync(lens, lens_restore_host, static_cast<size_t>(B) * 4, cudaMemcpyHostToDevice, st) !=
          cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    rc = SLIM_ECUDA;
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  cudaGetLastError();
  return rc;
}

}  // extern "C"
