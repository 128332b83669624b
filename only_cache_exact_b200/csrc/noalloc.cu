// slim_decode_step_noalloc: the generation step for callers that cannot
// allocate device memory. Some hosts hand a plug-in only the buffers it
// computes on: an inference runtime that owns every byte of device memory
// under a plan fixed at start-up, or a latency-critical decode loop in which
// cudaMalloc's implicit device synchronisation is not acceptable. Such a
// caller cannot provide the workspace slim_decode_step needs, so this entry
// point takes its scratch from a fixed buffer compiled into this library.
#include <cuda_runtime.h>

#include <mutex>

#include "slim_internal.h"

// Scratch of the allocation-free entry point: SLIM_NOALLOC_SCRATCH_BYTES bytes
// on every GPU that loads this library, held until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SLIM_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch buffer on the current device. In host code
// g_noalloc_scratch names a host-side stand-in, not device memory, so the
// address is looked up once per device with that device current.
int scratch_on_current_device(void** addr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return SLIM_ECUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return SLIM_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return SLIM_ECUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *addr = g_scratch_addr[dev];
  return SLIM_OK;
}

}  // namespace

extern "C" size_t slim_noalloc_scratch_bytes(void) { return static_cast<size_t>(SLIM_NOALLOC_SCRATCH_BYTES); }

extern "C" int slim_decode_step_noalloc(const float* q, const void* k_new, void* Kcache, int32_t* lens,
                                        const void* W_KV, int dtype, int B, int d, int H, int64_t cap, int variant,
                                        int64_t t_hint, float* out, int32_t* dev_status, void* stream) {
  const size_t need = slim_decode_workspace_bytes(dtype, B, d, H, cap, variant);
  if (need == 0) return SLIM_EINVAL;
  if (need > static_cast<size_t>(SLIM_NOALLOC_SCRATCH_BYTES)) return SLIM_EWORKSPACE;
  void* scratch = nullptr;
  const int rc = scratch_on_current_device(&scratch);
  if (rc != SLIM_OK) return rc;
  return slim_decode_step(q, k_new, Kcache, lens, W_KV, dtype, B, d, H, cap, variant, t_hint, out, scratch,
                          static_cast<size_t>(SLIM_NOALLOC_SCRATCH_BYTES), dev_status, stream);
}
