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

#include <algorithm>

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
  int32_t* status;
  int B, d, H, ndb, max_items;
  int sb;           // sequences per cluster reduction round
};

constexpr int kReduceThreads = 256;
constexpr int kReduceNBB = 8;  // sequences per projection block (register accumulators)

template <typename WT>
struct WVec;
template <>
struct WVec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void load(const __nv_bfloat16* p, float (&w)[8]) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
    w[0] = bf16lo(v.x); w[1] = bf16hi(v.x); w[2] = bf16lo(v.y); w[3] = bf16hi(v.y);
    w[4] = bf16lo(v.z); w[5] = bf16hi(v.z); w[6] = bf16lo(v.w); w[7] = bf16hi(v.w);
  }
};
template <>
struct WVec<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void load(const float* p, float (&w)[4]) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(p));
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  }
};

struct ReduceSmem {
  uint32_t wts, ubar, part, red, total;
};
__host__ __device__ inline ReduceSmem reduce_smem_layout(int max_items, int DB, int d_h, int sb) {
  ReduceSmem r;
  uint32_t o = 0;
  r.wts = o;
  o += ((static_cast<uint32_t>(max_items) + 3u) & ~3u) * 4u;
  r.ubar = o;
  o += static_cast<uint32_t>(kReduceNBB) * DB * 4u;
  r.part = o;
  o += static_cast<uint32_t>(sb) * d_h * 4u;
  r.red = o;
  o += static_cast<uint32_t>(kReduceThreads / 32) * kReduceNBB * d_h * 4u;
  r.total = o;
  return r;
}

template <typename WT>
__global__ void __launch_bounds__(kReduceThreads) reduce_b_kernel(const ReduceBParams p) {
  extern __shared__ __align__(16) uint8_t rsm[];
  constexpr int VEC = WVec<WT>::N;
  const int h = blockIdx.x, r = blockIdx.y;
  const int d_h = p.d / p.H;
  const int DB = p.d / p.ndb, c0 = r * DB;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const WT* W = static_cast<const WT*>(p.w_kv);
  const ReduceSmem L = reduce_smem_layout(p.max_items, DB, d_h, p.sb);
  float* wts = reinterpret_cast<float*>(rsm + L.wts);
  float* ubar = reinterpret_cast<float*>(rsm + L.ubar);
  float* part = reinterpret_cast<float*>(rsm + L.part);
  float* red = reinterpret_cast<float*>(rsm + L.red);

  // Before the partials exist: pull this CTA's W_KV block (rows c0.., head-h columns) into L2.
  {
    const int row_bytes = d_h * static_cast<int>(sizeof(WT));
    const int lines = (row_bytes + 127) / 128;
    for (int i = tid; i < DB * lines; i += kReduceThreads) {
      const int row = i / lines, ln = i % lines;
      const char* a = reinterpret_cast<const char*>(W + static_cast<size_t>(c0 + row) * p.d + h * d_h) + ln * 128;
      asm volatile("prefetch.global.L2 [%0];" ::"l"(a));
    }
  }
  pdl_wait_primary();
  pdl_launch_dependents();
  __syncthreads();

  const int32_t* off = p.meta + 1;
  if (h == 0 && r == 0) {
    for (int b = tid; b < p.B; b += kReduceThreads)
      if (p.meta[2 + p.B + b] & kSeqAppend) p.lens[b] += 1;
  }

  // merge weights 2^(m_c - M) / L of every item c for head h
  for (int b = warp; b < p.B; b += kReduceThreads / 32) {
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
  __syncthreads();

  const int ncg = d_h / VEC;               // column groups of VEC columns
  const int G = kReduceThreads / ncg;      // row groups
  const int cg = tid % ncg, g = tid / ncg;
  const int gpw = 32 / ncg;                // row groups per warp (ncg <= 32)
  const uint32_t part_base = smem_u32(part);

  for (int s0 = 0; s0 < p.B; s0 += p.sb) {
    const int nsb = min(p.sb, p.B - s0);
    for (int b0 = s0; b0 < s0 + nsb; b0 += kReduceNBB) {
      const int nbb = min(kReduceNBB, s0 + nsb - b0);
      // ū of the block straight from the partials: float4 loads, eight items in flight per thread
      const int nv = DB / 4;
      const size_t item4 = static_cast<size_t>(p.H) * p.d / 4;  // float4 stride between items
      for (int i = tid; i < kReduceNBB * nv; i += kReduceThreads) {
        const int bl = i / nv, c4 = i % nv;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (bl < nbb) {
          const int lo = off[b0 + bl], hi = off[b0 + bl + 1];
          const float4* src =
              reinterpret_cast<const float4*>(p.U + (static_cast<size_t>(lo) * p.H + h) * p.d + c0) + c4;
          int c = lo;
          for (; c + 8 <= hi; c += 8) {
            float4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = __ldg(src + u * item4);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const float w = wts[c + u];
              acc.x = fmaf(w, v[u].x, acc.x);
              acc.y = fmaf(w, v[u].y, acc.y);
              acc.z = fmaf(w, v[u].z, acc.z);
              acc.w = fmaf(w, v[u].w, acc.w);
            }
            src += 8 * item4;
          }
          for (; c < hi; ++c, src += item4) {
            const float4 v = __ldg(src);
            const float w = wts[c];
            acc.x = fmaf(w, v.x, acc.x);
            acc.y = fmaf(w, v.y, acc.y);
            acc.z = fmaf(w, v.z, acc.z);
            acc.w = fmaf(w, v.w, acc.w);
          }
        }
        *reinterpret_cast<float4*>(ubar + bl * DB + 4 * c4) = acc;
      }
      __syncthreads();
      // partial head output of the block: ū[bl, d-block] · W_KV[d-block rows, head-h columns]
      float acc[kReduceNBB][VEC];
#pragma unroll
      for (int bl = 0; bl < kReduceNBB; ++bl)
#pragma unroll
        for (int v = 0; v < VEC; ++v) acc[bl][v] = 0.f;
      if (g < G) {
        const WT* wp = W + static_cast<size_t>(c0) * p.d + h * d_h + cg * VEC;
#pragma unroll 4
        for (int i = g; i < DB; i += G) {
          float w[VEC];
          WVec<WT>::load(wp + static_cast<size_t>(i) * p.d, w);
#pragma unroll
          for (int bl = 0; bl < kReduceNBB; ++bl) {
            const float u = ubar[bl * DB + i];
#pragma unroll
            for (int v = 0; v < VEC; ++v) acc[bl][v] = fmaf(u, w[v], acc[bl][v]);
          }
        }
      }
      // reduce the row groups of a warp with shuffles, then across warps through shared memory
#pragma unroll
      for (int bl = 0; bl < kReduceNBB; ++bl)
#pragma unroll
        for (int v = 0; v < VEC; ++v)
          for (int o = ncg; o < 32; o <<= 1) acc[bl][v] += __shfl_xor_sync(0xffffffffu, acc[bl][v], o);
      if (lane < ncg && g < G) {
#pragma unroll
        for (int bl = 0; bl < kReduceNBB; ++bl)
#pragma unroll
          for (int v = 0; v < VEC; ++v) red[(warp * kReduceNBB + bl) * d_h + cg * VEC + v] = acc[bl][v];
      }
      __syncthreads();
      const int nwarps = min(kReduceThreads / 32, (G + gpw - 1) / gpw);
      for (int i = tid; i < nbb * d_h; i += kReduceThreads) {
        float sum = 0.f;
        for (int w2 = 0; w2 < nwarps; ++w2) sum += red[w2 * kReduceNBB * d_h + i];
        part[(b0 - s0) * d_h + i] = sum;
      }
      __syncthreads();
    }
    // sum the NDB CTAs' products through distributed shared memory (fixed order)
    cluster_sync();
    for (int i = tid; i < nsb * d_h; i += kReduceThreads) {
      if (i % p.ndb != r) continue;
      float sum = 0.f;
      for (int q = 0; q < p.ndb; ++q) sum += ld_cluster_f32(mapa_shared(part_base + 4u * i, q));
      const int bl = i / d_h, jj = i % d_h;
      p.out[static_cast<size_t>(s0 + bl) * p.d + h * d_h + jj] = sum;
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
  const int vec = (a.dtype == SLIM_BF16) ? 8 : 4;
  if (d_h % vec || d_h / vec > 32 || (32 % (d_h / vec)) != 0) return cudaErrorNotSupported;
  ReduceBParams p;
  p.U = ws.U;
  p.m = ws.m;
  p.l = ws.l;
  p.meta = ws.meta;
  p.w_kv = a.w_kv;
  p.out = a.out;
  p.lens = a.lens;
  p.status = a.status;
  p.B = a.B;
  p.d = a.d;
  p.H = a.H;
  p.ndb = pick_ndb(a.d, d_h);
  p.max_items = ws.max_items;
  const int DB = a.d / p.ndb;
  if (DB % 4) return cudaErrorNotSupported;
  p.sb = std::max(kReduceNBB, std::min(a.B, (32 * 1024) / (d_h * 4)) / kReduceNBB * kReduceNBB);
  p.sb = std::min(p.sb, ((a.B + kReduceNBB - 1) / kReduceNBB) * kReduceNBB);
  const size_t smem = reduce_smem_layout(p.max_items, DB, d_h, p.sb).total;
  if (smem > 200u * 1024u) return cudaErrorNotSupported;
  auto kern = (a.dtype == SLIM_BF16) ? reduce_b_kernel<__nv_bfloat16> : reduce_b_kernel<float>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.H), static_cast<unsigned>(p.ndb), 1);
  cfg.blockDim = dim3(kReduceThreads, 1, 1);
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
