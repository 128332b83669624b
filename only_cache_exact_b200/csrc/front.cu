// Step front end: q = x·W_Q and k = x·W_K for the B input rows of one generation step.
//
// Slim Attention article, section "K-Cache is All You Need", generation phase:
// a step starts from the new token's input row x; its query q = x·W_Q is scored
// against the cached keys, and (self-attention) its key k = x·W_K is appended to
// the K cache; a cross-attention step needs q only. Row vectors: W is stored
// [d_in][d_out] row-major and multiplied from the right.
//
// front_tc_kernel (bf16, d a multiple of 128): a CTA owns 128 output columns of
// W_Q or W_K for up to 256 rows of x and a contiguous share of the reduction;
// clusters of KS CTAs split the reduction when there are too few column tiles
// to occupy the SMs, and sum their fp32 partial tiles in rank order through
// distributed shared memory (so the result does not depend on timing).
//   warp 0     TMA producer: 64x128 tiles of W (two 64-column blocks) and
//              64-column tiles of the Bp rows of x (Bp = B rounded up to 16,
//              rows past B read as zero), 128-byte swizzle, a ring of 4..8
//              stages; W streams evict-first (read once), x evict-last (read
//              by every column tile)
//   warp 1     tcgen05.mma M=128 (output columns) N=Bp (rows of x) K=16 into
//              a Bp-column fp32 TMEM accumulator; W is the MN-major A operand
//              read in place, x the K-major B operand
//   warps 2-5  accumulator (TMEM lane = column) -> q (fp32) or k (bf16,
//              rounded once) or the cluster's partial tile
// The work is bound by reading W once: 2·d² bytes per projection.
//
// front_simt_kernel (fp32, and bf16 shapes without a 128-column tiling): one
// thread per output column and up to 8 rows, one fp32 accumulator per output
// with the fused multiply-adds in ascending order of the reduction index, so
// the fp32 result is fixed bit for bit.
#include <cuda_bf16.h>

#include <algorithm>

#include "slim_internal.h"
#include "ptx.cuh"

namespace slim {

namespace {

constexpr int kFM = 128, kFK = 64, kFThreads = 192, kFMaxRows = 256;
constexpr uint32_t kFW = kFK * kFM * 2;    // W tile: 64 rows x 128 columns, 16 KB
constexpr uint32_t kFRingMax = 200u << 10;  // bytes of the W and x rings

__host__ __device__ inline uint32_t front_xbytes(int Bp) { return static_cast<uint32_t>(Bp) * 128u; }
__host__ __device__ inline int front_stages(int Bp) {
  const int s = static_cast<int>(kFRingMax / (kFW + front_xbytes(Bp)));
  return s > 8 ? 8 : s;  // >= 4 for Bp <= 256
}
__host__ __device__ inline uint32_t front_smem(int Bp) {
  return static_cast<uint32_t>(front_stages(Bp)) * (kFW + front_xbytes(Bp)) + 256u + 1024u;
}

struct FrontParams {
  float* q;           // [B][d]
  __nv_bfloat16* k;   // [B][d], null for a cross-attention step
  int B, d;
  int qtiles;         // d / 128: column tiles [0, qtiles) are W_Q's, the rest W_K's
  int nk;             // d / 64 reduction chunks
  int Bp;             // rows of x per CTA (B rounded up to 16, at most 256)
  uint32_t tmem_cols; // accumulator columns allocated (power of two >= max(32, Bp))
};

__device__ __forceinline__ float to_float(float v) { return v; }
__device__ __forceinline__ float to_float(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T>
__device__ __forceinline__ T from_float(float v) {
  return v;
}
template <>
__device__ __forceinline__ __nv_bfloat16 from_float<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

__device__ __forceinline__ void front_store(const FrontParams& p, bool is_q, int b, int col, float a) {
  const size_t o = static_cast<size_t>(b) * p.d + col;
  if (is_q) p.q[o] = a;
  else p.k[o] = __float2bfloat16_rn(a);
}

template <int KS>
__global__ void __launch_bounds__(kFThreads, 1)
    front_tc_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap wqmap,
                    const __grid_constant__ CUtensorMap wkmap, const FrontParams p, int32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int Bp = p.Bp, stages = front_stages(Bp);
  const uint32_t xb = front_xbytes(Bp);
  uint8_t* wsm = smem;                       // [stages][2 column blocks][64 rows][128 B]
  uint8_t* xs = smem + stages * kFW;         // [stages][Bp rows][128 B]
  float* red = reinterpret_cast<float*>(smem);  // after the main loop: the partial tile [Bp][128]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + stages * (kFW + xb));
  uint64_t* empty = full + stages;
  uint64_t* accfull = empty + stages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accfull + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x / KS;
  const int kr = KS > 1 ? static_cast<int>(cluster_ctarank()) : 0;
  const bool is_q = tile < p.qtiles;
  const int n0 = (is_q ? tile : tile - p.qtiles) * kFM;  // first column within W_Q or W_K
  const int m0 = blockIdx.y * kFMaxRows;                  // first row of x
  const int kper = p.nk / KS, kc0 = kr * kper;            // this CTA's reduction chunks
  const CUtensorMap* wmap = is_q ? &wqmap : &wkmap;

  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&xmap);
    tma_prefetch_desc(wmap);
  } else if (warp == 1) {
    if (lane == 0) {
      for (int s = 0; s < stages; ++s) {
        mbar_init(&full[s], 1);
        mbar_init(&empty[s], 1);
      }
      mbar_init(accfull, 1);
      fence_barrier_init();
    }
    __syncwarp();
    tmem_alloc(tmem_slot, p.tmem_cols);
    tmem_relinquish();
  }
  // Launched as a programmatic dependent: nothing above touched global memory; x, the weights
  // and the outputs are accessed only after the previous kernel in the stream has completed.
  // The step's split kernel may then be scheduled at once (it waits for this grid itself).
  pdl_wait_primary();
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_x = l2_policy_evict_last();
      const uint64_t pol_w = l2_policy_evict_first();
      int g = 0;
      for (; g < kper; ++g) {
        const int s = g % stages;
        const uint32_t ph = static_cast<uint32_t>(g / stages) & 1u;
        if (g >= stages && !mbar_wait(&empty[s], ph ^ 1u, status)) break;
        mbar_arrive_expect_tx(&full[s], kFW + xb);
        const int kc = (kc0 + g) * kFK;
        tma_load_3d(wsm + s * kFW, wmap, 0, kc, n0 / 64, &full[s], pol_w);
        tma_load_2d(xs + s * xb, &xmap, kc, m0, &full[s], pol_x);
      }
      for (int t = max(0, g - stages); t < g; ++t)  // every issued copy lands before the CTA exits
        mbar_wait(&full[t % stages], static_cast<uint32_t>(t / stages) & 1u, status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kFM, static_cast<uint32_t>(Bp), 1u, 0u);
      const uint32_t wbase = smem_u32(wsm), xbase = smem_u32(xs);
      for (int g = 0; g < kper; ++g) {
        const int s = g % stages;
        if (!mbar_wait(&full[s], static_cast<uint32_t>(g / stages) & 1u, status)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kFK / 16; ++kk) {
          // W: MN-major, 64-column blocks 8 KB apart, 8-row groups 1024 B apart, 16 rows per step
          const uint64_t ad = smem_desc(wbase + s * kFW + kk * 16 * 128, kFK * 128, 1024, kLayoutSW128);
          // x: K-major, 8-row groups 1024 B apart, a 16-element step is 32 B into the swizzled row
          const uint64_t bd = smem_desc(xbase + s * xb + kk * 32, 16, 1024, kLayoutSW128);
          umma_f16(tmem, ad, bd, idesc, (g > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&empty[s]);
      }
      umma_commit(accfull);  // also after a failed wait: covers every MMA issued
      mbar_wait(accfull, 0u, status);
    }
  } else {
    // TMEM lane = output column of the tile (warps 2..5 take lane quarters 2, 3, 0, 1), TMEM
    // column = row of x
    const int quarter = warp & 3;
    const int col = quarter * 32 + lane;
    const bool got = __all_sync(0xffffffffu, mbar_wait(accfull, 0u, status));
    tc_fence_after();
    const int nrows = min(Bp, p.B - m0);
    const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    for (int r0 = 0; r0 < nrows; r0 += 16) {
      float v[16];
      if (got) {
        tmem_ld16(taddr + static_cast<uint32_t>(r0), v);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = 0.f;
      }
      if constexpr (KS == 1) {
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (r0 + i < nrows) front_store(p, is_q, m0 + r0 + i, n0 + col, v[i]);
      } else {
        // the ring is free: every copy has landed and every MMA has completed (accfull)
#pragma unroll
        for (int i = 0; i < 16; ++i) red[(r0 + i) * kFM + col] = v[i];
      }
    }
  }
  __syncwarp();  // lanes 1..31 of warps 0 and 1 skipped the lane-0 loops
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, p.tmem_cols);
  }
  if constexpr (KS > 1) {
    // CTA kr of the cluster finishes columns [kr·128/KS, (kr+1)·128/KS): the partial tiles of
    // ranks 0 .. KS-1 added in that order
    cluster_sync();
    constexpr int cw = kFM / KS;
    const int nrows = min(Bp, p.B - m0);
    const uint32_t rbase = smem_u32(red);
    for (int e = threadIdx.x; e < nrows * cw; e += kFThreads) {
      const int r = e / cw, c = kr * cw + e % cw;
      const uint32_t off = 4u * static_cast<uint32_t>(r * kFM + c);
      float a = 0.f;
#pragma unroll
      for (int s = 0; s < KS; ++s) a += ld_cluster_f32(mapa_shared(rbase + off, static_cast<uint32_t>(s)));
      front_store(p, is_q, m0 + r, n0 + c, a);
    }
    cluster_sync();  // no CTA exits while a peer may still read its partial tile
  }
}

constexpr int kSRows = 8, kSCols = 128, kSChunk = 256;

template <typename T>
__global__ void __launch_bounds__(kSCols) front_simt_kernel(const T* __restrict__ x, const T* __restrict__ wq,
                                                            const T* __restrict__ wk, float* __restrict__ q,
                                                            T* __restrict__ k, int B, int d) {
  __shared__ float xs[kSRows][kSChunk];
  pdl_wait_primary();  // launched as a programmatic dependent: wait before any global access
  pdl_launch_dependents();
  const int col = blockIdx.x * kSCols + threadIdx.x;  // column of [W_Q | W_K]
  const int b0 = blockIdx.y * kSRows;
  const int nr = min(kSRows, B - b0);
  const bool is_q = col < d;
  const int j = is_q ? col : col - d;
  const bool active = col < (wk ? 2 * d : d);
  const T* W = is_q ? wq : wk;
  float acc[kSRows];
#pragma unroll
  for (int r = 0; r < kSRows; ++r) acc[r] = 0.f;
  for (int i0 = 0; i0 < d; i0 += kSChunk) {
    const int n = min(kSChunk, d - i0);
    __syncthreads();
    for (int e = threadIdx.x; e < kSRows * kSChunk; e += kSCols) {
      const int r = e / kSChunk, i = e % kSChunk;
      xs[r][i] = (r < nr && i < n) ? to_float(x[static_cast<size_t>(b0 + r) * d + i0 + i]) : 0.f;
    }
    __syncthreads();
    if (active) {
      for (int i = 0; i < n; ++i) {
        const float w = to_float(W[static_cast<size_t>(i0 + i) * d + j]);
#pragma unroll
        for (int r = 0; r < kSRows; ++r) acc[r] = __fmaf_rn(xs[r][i], w, acc[r]);
      }
    }
  }
  if (!active) return;
  for (int r = 0; r < nr; ++r) {
    const size_t o = static_cast<size_t>(b0 + r) * d + j;
    if (is_q) q[o] = acc[r];
    else k[o] = from_float<T>(acc[r]);
  }
}

template <int KS>
cudaError_t launch_front_tc(const CUtensorMap& xmap, const CUtensorMap& wqmap, const CUtensorMap& wkmap,
                            const FrontParams& p, int32_t* status, cudaStream_t st) {
  auto kern = front_tc_kernel<KS>;
  const uint32_t smem = front_smem(p.Bp);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int tiles = p.qtiles + (p.k ? p.qtiles : 0);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles * KS), static_cast<unsigned>((p.B + kFMaxRows - 1) / kFMaxRows), 1);
  cfg.blockDim = dim3(kFThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = KS;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = KS > 1 ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, xmap, wqmap, wkmap, p, status);
}

}  // namespace

bool front_tc_supported(int dtype, int d) { return dtype == SLIM_BF16 && d % kFM == 0; }

// Cluster size of the tensor-core front end: split the reduction until the column tiles fill the
// SMs, keeping at least two 64-row chunks per CTA.
int front_tc_split(int d, bool with_k) {
  const int tiles = (d / kFM) * (with_k ? 2 : 1), nk = d / kFK;
  for (int ks : {8, 4, 2})
    if (tiles * ks <= num_sms() && nk % ks == 0 && nk / ks >= 2) return ks;
  return 1;
}

cudaError_t launch_front(const void* x, const void* W_Q, const void* W_K, float* q, void* k, int dtype, int B, int d,
                         int32_t* status, cudaStream_t st, int* launches) {
  cudaError_t e;
  if (front_tc_supported(dtype, d)) {
    CUtensorMap xmap, wqmap, wkmap;
    const int Bp = std::min(kFMaxRows, (B + 15) & ~15);
    // x [B rows][d] with a 64 x Bp box; W as {64 columns, d rows, d/64 column blocks} with a
    // 64 x 64 x 2 box (a 64-row, 128-column tile)
    if (!encode_tmap_2d_bf16(&xmap, x, static_cast<uint64_t>(d), static_cast<uint64_t>(B),
                             static_cast<uint64_t>(d) * 2u, kFK, static_cast<uint32_t>(Bp), true) ||
        !encode_tmap_3d_bf16(&wqmap, W_Q, 64, static_cast<uint64_t>(d), static_cast<uint64_t>(d / 64),
                             static_cast<uint64_t>(d) * 2u, 128, 64, kFK, kFM / 64) ||
        !encode_tmap_3d_bf16(&wkmap, W_K ? W_K : W_Q, 64, static_cast<uint64_t>(d), static_cast<uint64_t>(d / 64),
                             static_cast<uint64_t>(d) * 2u, 128, 64, kFK, kFM / 64))
      return cudaErrorInvalidValue;
    uint32_t tcols = 32;
    while (tcols < static_cast<uint32_t>(Bp)) tcols <<= 1;
    FrontParams p{q, static_cast<__nv_bfloat16*>(W_K ? k : nullptr), B, d, d / kFM, d / kFK, Bp, tcols};
    const int ks = front_tc_split(d, W_K != nullptr);
    e = ks == 8   ? launch_front_tc<8>(xmap, wqmap, wkmap, p, status, st)
        : ks == 4 ? launch_front_tc<4>(xmap, wqmap, wkmap, p, status, st)
        : ks == 2 ? launch_front_tc<2>(xmap, wqmap, wkmap, p, status, st)
                  : launch_front_tc<1>(xmap, wqmap, wkmap, p, status, st);
  } else {
    const int cols = W_K ? 2 * d : d;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((cols + kSCols - 1) / kSCols), static_cast<unsigned>((B + kSRows - 1) / kSRows));
    cfg.blockDim = dim3(kSCols, 1, 1);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (dtype == SLIM_BF16)
      e = cudaLaunchKernelEx(&cfg, front_simt_kernel<__nv_bfloat16>, static_cast<const __nv_bfloat16*>(x),
                             static_cast<const __nv_bfloat16*>(W_Q), static_cast<const __nv_bfloat16*>(W_K), q,
                             static_cast<__nv_bfloat16*>(k), B, d);
    else
      e = cudaLaunchKernelEx(&cfg, front_simt_kernel<float>, static_cast<const float*>(x),
                             static_cast<const float*>(W_Q), static_cast<const float*>(W_K), q, static_cast<float*>(k),
                             B, d);
  }
  if (e == cudaSuccess && launches) ++*launches;
  return e;
}

}  // namespace slim
