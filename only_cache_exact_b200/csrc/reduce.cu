// Merge of the split-T partials and the W_KV projection.
//
// Ordering (b) (Slim Attention article, section "K-Cache is All You Need",
// second generation-phase option, with W_KV = W_K^(-1)·W_V): for sequence b
// and head h, the chunk partials (m_c, l_c, U_c) combine by the log-sum-exp
// rule into  ū = Σ_c 2^(m_c - M) U_c / Σ_c 2^(m_c - M) l_c,  M = max_c m_c,
// and the head output is  o[b, h-cols] = ū · W_KV[:, h-cols].
//
// Grid (H, NDB) with clusters of NDB CTAs along y: CTA (h, r) merges the
// d-block r of ū for every sequence and multiplies it by the matching
// d-block rows of W_KV's head-h columns; the NDB partial products are summed
// through distributed shared memory (deterministic order) and written once.
// The kernel is launched as a programmatic dependent of the split kernel: it
// prefetches its W_KV block into L2 before waiting for the partials.
//
// Ordering (a) needs only the merge (its partials are already softmax·V).
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace slim {

struct ReduceBParams {
  const float* U;
  const float* m;
  const float* l;
  const int32_t* meta;
  const void* w_kv;
  float* out;
  int32_t* lens;
  int B, d, H, ndb, bb, max_items;
};

template <typename WT>
__device__ __forceinline__ float ldw(const WT* w, size_t i);
template <>
__device__ __forceinline__ float ldw<float>(const float* w, size_t i) {
  return __ldg(w + i);
}
template <>
__device__ __forceinline__ float ldw<__nv_bfloat16>(const __nv_bfloat16* w, size_t i) {
  return __bfloat162float(w[i]);
}

template <typename WT>
__global__ void __launch_bounds__(256) reduce_b_kernel(const ReduceBParams p) {
  extern __shared__ float rsm[];
  const int h = blockIdx.x, r = blockIdx.y;
  const int d_h = p.d / p.H;
  const int DB = p.d / p.ndb, c0 = r * DB;
  const int tid = threadIdx.x;
  const WT* W = static_cast<const WT*>(p.w_kv);

  // Before the partials exist: pull this CTA's W_KV block into L2.
  {
    const int row_bytes = d_h * static_cast<int>(sizeof(WT));
    const int lines = (row_bytes + 127) / 128;
    for (int i = tid; i < DB * lines; i += blockDim.x) {
      const int row = i / lines, ln = i % lines;
      const char* a = reinterpret_cast<const char*>(W + static_cast<size_t>(c0 + row) * p.d + h * d_h) + ln * 128;
      asm volatile("prefetch.global.L2 [%0];" ::"l"(a));
    }
  }
  pdl_wait_primary();

  const int items = p.meta[0];
  const int32_t* off = p.meta + 1;
  float* wts = rsm;                         // [max_items]
  float* ubar = wts + p.max_items;          // [bb][DB]
  float* part = ubar + p.bb * DB;           // [bb][d_h]
  float* red = part + p.bb * d_h;           // [groups][bb][d_h]

  if (h == 0 && r == 0) {
    for (int b = tid; b < p.B; b += blockDim.x)
      if (p.meta[2 + p.B + b] & kSeqAppend) p.lens[b] += 1;
  }

  // merge weights 2^(m_c - M) / L for every item of head h
  const int warp = tid >> 5, lane = tid & 31, nw = blockDim.x >> 5;
  for (int b = warp; b < p.B; b += nw) {
    const int c_lo = off[b], c_hi = off[b + 1];
    float M = -INFINITY;
    for (int c = c_lo + lane; c < c_hi; c += 32) M = fmaxf(M, p.m[static_cast<size_t>(c) * p.H + h]);
    M = warp_max(M);
    float Ls = 0.f;
    for (int c = c_lo + lane; c < c_hi; c += 32)
      Ls += exp2f(p.m[static_cast<size_t>(c) * p.H + h] - M) * p.l[static_cast<size_t>(c) * p.H + h];
    Ls = warp_sum(Ls);
    const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
    for (int c = c_lo + lane; c < c_hi; c += 32) wts[c] = exp2f(p.m[static_cast<size_t>(c) * p.H + h] - M) * inv;
  }
  (void)items;
  __syncthreads();

  const int groups = blockDim.x / d_h;  // d_h <= 256
  const int j = tid % d_h, g = tid / d_h;
  const uint32_t part_base = smem_u32(part);

  for (int b0 = 0; b0 < p.B; b0 += p.bb) {
    const int nbb = min(p.bb, p.B - b0);
    // ū for the d-block of this CTA
    for (int i = tid; i < nbb * DB; i += blockDim.x) {
      const int bl = i / DB, col = i % DB;
      const int b = b0 + bl;
      float acc = 0.f;
      for (int c = off[b]; c < off[b + 1]; ++c)
        acc = fmaf(wts[c], p.U[(static_cast<size_t>(c) * p.H + h) * p.d + c0 + col], acc);
      ubar[bl * DB + col] = acc;
    }
    __syncthreads();
    // partial head output: ū[bl, block] · W_KV[block, h-cols]
    if (g < groups) {
      float acc[16];
#pragma unroll
      for (int bl = 0; bl < 16; ++bl) acc[bl] = 0.f;
      for (int i = g; i < DB; i += groups) {
        const float w = ldw<WT>(W, static_cast<size_t>(c0 + i) * p.d + h * d_h + j);
#pragma unroll
        for (int bl = 0; bl < 16; ++bl)
          if (bl < nbb) acc[bl] = fmaf(ubar[bl * DB + i], w, acc[bl]);
      }
#pragma unroll
      for (int bl = 0; bl < 16; ++bl)
        if (bl < nbb) red[(g * p.bb + bl) * d_h + j] = acc[bl];
    }
    __syncthreads();
    for (int i = tid; i < nbb * d_h; i += blockDim.x) {
      float s = 0.f;
      for (int gg = 0; gg < groups; ++gg) s += red[gg * p.bb * d_h + i];
      part[i] = s;
    }
    // sum the NDB CTAs' products through distributed shared memory
    cluster_sync();
    for (int i = tid; i < nbb * d_h; i += blockDim.x) {
      if (i % p.ndb != r) continue;
      float s = 0.f;
      for (int rr = 0; rr < p.ndb; ++rr) s += ld_cluster_f32(mapa_shared(part_base + 4u * i, rr));
      const int bl = i / d_h, jj = i % d_h;
      p.out[static_cast<size_t>(b0 + bl) * p.d + h * d_h + jj] = s;
    }
    cluster_sync();
  }
}

// ---------------------------------------------------------------------------- ordering (a) merge
struct ReduceAParams {
  const float* O;
  const float* m;
  const float* l;
  const int32_t* meta;
  float* out;
  int32_t* lens;
  int B, d, H;
};

__global__ void __launch_bounds__(256) reduce_a_kernel(const ReduceAParams p) {
  const int b = blockIdx.x;
  const int d_h = p.d / p.H;
  const int32_t* off = p.meta + 1;
  const int c_lo = off[b], c_hi = off[b + 1];
  if (b == 0 && threadIdx.x == 0) {
    for (int s = 0; s < p.B; ++s)
      if (p.meta[2 + p.B + s] & kSeqAppend) p.lens[s] += 1;
  }
  for (int col = threadIdx.x; col < p.d; col += blockDim.x) {
    const int h = col / d_h;
    float M = -INFINITY;
    for (int c = c_lo; c < c_hi; ++c) M = fmaxf(M, p.m[static_cast<size_t>(c) * p.H + h]);
    float Ls = 0.f, acc = 0.f;
    for (int c = c_lo; c < c_hi; ++c) {
      const float w = exp2f(p.m[static_cast<size_t>(c) * p.H + h] - M);
      Ls = fmaf(w, p.l[static_cast<size_t>(c) * p.H + h], Ls);
      acc = fmaf(w, p.O[static_cast<size_t>(c) * p.d + col], acc);
    }
    p.out[static_cast<size_t>(b) * p.d + col] = Ls > 0.f ? acc / Ls : 0.f;
  }
}

// ---------------------------------------------------------------------------- host
namespace {
int pick_ndb(int d, int d_h) {
  // d-blocks per head: a cluster of up to 8 CTAs; blocks stay multiples of 8 columns.
  for (int n = 8; n >= 1; --n)
    if (d % n == 0 && (d / n) % 8 == 0) return n;
  return 1;
}
}  // namespace

cudaError_t launch_reduce_b(const DecodeArgs& a, const SplitWorkspace& ws, bool pdl, cudaStream_t st,
                            int* launches) {
  const int d_h = a.d / a.H;
  if (d_h > 256) return cudaErrorNotSupported;
  ReduceBParams p;
  p.U = ws.U;
  p.m = ws.m;
  p.l = ws.l;
  p.meta = ws.meta;
  p.w_kv = a.w_kv;
  p.out = a.out;
  p.lens = a.lens;
  p.B = a.B;
  p.d = a.d;
  p.H = a.H;
  p.ndb = pick_ndb(a.d, d_h);
  p.max_items = ws.max_items;
  const int DB = a.d / p.ndb;
  const int groups = 256 / d_h;
  p.bb = 16;
  size_t smem = 0;
  for (;;) {
    smem = sizeof(float) * (static_cast<size_t>(p.max_items) + static_cast<size_t>(p.bb) * DB +
                            static_cast<size_t>(p.bb) * d_h + static_cast<size_t>(groups) * p.bb * d_h);
    if (smem <= 200 * 1024 || p.bb == 1) break;
    p.bb /= 2;
  }
  if (smem > 200 * 1024) return cudaErrorNotSupported;
  auto kern = (a.dtype == SLIM_BF16) ? reduce_b_kernel<__nv_bfloat16> : reduce_b_kernel<float>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.H), static_cast<unsigned>(p.ndb), 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = static_cast<unsigned>(p.ndb);
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, kern, p);
  if (e == cudaSuccess && launches) ++*launches;
  return e;
}

cudaError_t launch_reduce_a(const DecodeArgs& a, const SplitWorkspace& ws, cudaStream_t st, int* launches) {
  ReduceAParams p;
  p.O = ws.U;
  p.m = ws.m;
  p.l = ws.l;
  p.meta = ws.meta;
  p.out = a.out;
  p.lens = a.lens;
  p.B = a.B;
  p.d = a.d;
  p.H = a.H;
  reduce_a_kernel<<<a.B, 256, 0, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess && launches) ++*launches;
  return e;
}

}  // namespace slim
