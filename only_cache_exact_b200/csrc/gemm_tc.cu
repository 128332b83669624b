// Prompt-phase projection K = X·W_K (and V = K·W_KV rows for ordering (a)):
// length bookkeeping after the projection kernels.
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace slim {

// lens[b] += n where the n new rows fitted (lens[b] + n <= cap); otherwise the
// projection kernels skipped the sequence and the status word records why.
__global__ void advance_lens_kernel(int32_t* lens, int B, int n, int64_t cap, int32_t* status) {
  int bad = 0;
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    const int L = lens[b];
    if (L < 0 || static_cast<int64_t>(L) > cap) bad |= SLIM_DEV_BADLEN;
    else if (static_cast<int64_t>(L) + n > cap) bad |= SLIM_DEV_OVERFLOW;
    else lens[b] = L + n;
  }
  if (bad) atomicOr(status, bad);
}

cudaError_t launch_advance_lens(int32_t* lens, int B, int n, int64_t cap, int32_t* status, cudaStream_t st,
                                int* launches) {
  advance_lens_kernel<<<1, 256, 0, st>>>(lens, B, n, cap, status);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess && launches) ++*launches;
  return e;
}

bool gemm_tc_supported(int d) {
  (void)d;
  return false;
}

cudaError_t launch_prefill_tc(const void*, const void*, void*, const int32_t*, int, int, int, int64_t, cudaStream_t,
                              int*) {
  return cudaErrorNotSupported;
}

cudaError_t launch_rows_gemm_tc(const void*, const void*, void*, const int32_t*, int, int, int, int64_t,
                                cudaStream_t, int*) {
  return cudaErrorNotSupported;
}

}  // namespace slim
