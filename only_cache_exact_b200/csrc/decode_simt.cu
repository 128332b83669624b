// CUDA-core kernels of the decode step and the row GEMM.
//
//  * decode_b_simt_kernel  ordering (b) split-T partials for any cache type
//                          (the fp32 workloads, and bf16 shapes without a
//                          tcgen05 configuration); exact online softmax.
//  * decode_a_simt_kernel  ordering (a) split-T partials over K (scores) and
//                          the materialised V = K·W_KV (values).
//  * append_kernel         writes this step's k at row lens[b] (ordering (a)).
//  * rows_gemm_kernel      Y_row = X_row · W with one fp32 accumulator per
//                          output, k ascending, one fused multiply-add per step;
//                          used for the fp32 prompt-phase projection K = X·W_K
//                          (bitwise equal to that order on any machine) and for
//                          V = K·W_KV of ordering (a).
// Source: Slim Attention article, section "K-Cache is All You Need" (prompt
// phase caches K = X·W_K; generation phase orderings (a) and (b)).
#include <cuda_bf16.h>

#include "split_plan.cuh"

namespace slim {

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T>
__device__ __forceinline__ T from_f(float v);
template <>
__device__ __forceinline__ float from_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

struct SimtParams {
  const float* q;
  const void* k_new;
  void* kcache;
  const void* vbuf;  // ordering (a): V rows, same layout as the cache
  const int32_t* lens;
  int32_t* status;
  float* ws_U;
  float* ws_m;
  float* ws_l;
  int32_t* ws_meta;
  int B, d, H;
  int64_t cap;
  int append;      // ordering (b): append k_new inside the kernel
  int attend_add;  // rows attended = lens[b] + attend_add
  int n_slots;
  int min_rows;
  float scale_log2;
};

constexpr int kSimtRows = 8;

// Shared memory of the SIMT decode kernels.
// (K and V tiles are staged in the cache's own element type, esize bytes.)
__host__ __device__ inline size_t simt_smem_bytes(int d, int H, int B, bool with_v, int esize) {
  const size_t tiles = static_cast<size_t>(kSimtRows) * d * esize * (with_v ? 2 : 1);
  size_t f = static_cast<size_t>(d)                      // q
             + static_cast<size_t>(with_v ? d : H * d)   // accumulator
             + 2 * static_cast<size_t>(H) * kSimtRows    // scores, p
             + 3 * static_cast<size_t>(H);               // m, l, alpha
  return f * 4 + ((tiles + 15) & ~size_t(15)) + (3 * static_cast<size_t>(B + 1) + 2) * 4 + 16;
}

template <typename KT, bool VARIANT_A>
__global__ void __launch_bounds__(256) decode_simt_kernel(const SimtParams p) {
  extern __shared__ float sm[];
  const int d = p.d, H = p.H, d_h = d / H;
  float* q_s = sm;
  float* acc = q_s + d;
  float* sc_base = acc + (VARIANT_A ? d : H * d);
  KT* ks = reinterpret_cast<KT*>(sc_base + 2 * H * kSimtRows + 3 * H);
  KT* vs = ks + kSimtRows * d;
  float* sc = sc_base;
  float* pm = sc + H * kSimtRows;
  float* mref = pm + H * kSimtRows;
  float* lsum = mref + H;
  float* alph = lsum + H;
  int* s_nb = reinterpret_cast<int*>(
      (reinterpret_cast<uintptr_t>(ks + kSimtRows * d * (VARIANT_A ? 2 : 1)) + 15) & ~uintptr_t(15));
  unsigned* s_q = reinterpret_cast<unsigned*>(s_nb + (p.B + 1));
  unsigned* s_soff = s_q + (p.B + 1);
  unsigned* s_plan = s_soff + (p.B + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (warp == 0)
    plan_lean(p.lens, p.B, 1, p.cap, p.attend_add, p.n_slots, p.min_rows, s_nb, s_q, s_soff, s_plan, p.ws_meta,
              p.status, blockIdx.x == 0);
  __syncthreads();
  LeanCursor cur;  // this CTA's segments
  cur.init(blockIdx.x, p.B, s_q, s_plan);
  SplitItem it;
  while (cur.next(it, s_nb, s_q, s_soff)) {
    const int b = it.b;
    const int nb_old = it.nb - p.append;
    const KT* K = static_cast<const KT*>(p.kcache) + static_cast<size_t>(b) * p.cap * d;
    const KT* V = static_cast<const KT*>(p.vbuf) + static_cast<size_t>(b) * p.cap * d;
    const KT* kn = static_cast<const KT*>(p.k_new) + static_cast<size_t>(b) * d;

    for (int i = tid; i < d; i += blockDim.x) q_s[i] = p.q[static_cast<size_t>(b) * d + i];
    const int nacc = VARIANT_A ? d : H * d;
    for (int i = tid; i < nacc; i += blockDim.x) acc[i] = 0.f;
    for (int h = tid; h < H; h += blockDim.x) {
      mref[h] = -INFINITY;
      lsum[h] = 0.f;
    }
    __syncthreads();

    for (int r_lo = it.row0; r_lo < it.row1; r_lo += kSimtRows) {
      const int nvalid = min(kSimtRows, it.row1 - r_lo);
      for (int i = tid; i < kSimtRows * d; i += blockDim.x) {
        const int row = i / d, col = i % d;
        const int r = r_lo + row;
        KT kv = from_f<KT>(0.f), vv = from_f<KT>(0.f);
        if (row < nvalid) {
          if (!VARIANT_A && p.append && r == nb_old) {
            kv = kn[col];
            static_cast<KT*>(p.kcache)[(static_cast<size_t>(b) * p.cap + r) * d + col] = kv;
          } else {
            kv = K[static_cast<size_t>(r) * d + col];
          }
          if (VARIANT_A) vv = V[static_cast<size_t>(r) * d + col];
        }
        ks[i] = kv;
        if (VARIANT_A) vs[i] = vv;
      }
      __syncthreads();
      // scores: warp w takes row w of the tile, every head
      if (warp < kSimtRows) {
        for (int h = 0; h < H; ++h) {
          float s = 0.f;
          for (int j = lane; j < d_h; j += 32) s = fmaf(q_s[h * d_h + j], to_f<KT>(ks[warp * d + h * d_h + j]), s);
          s = warp_sum(s);
          if (lane == 0) sc[h * kSimtRows + warp] = (warp < nvalid) ? s * p.scale_log2 : -INFINITY;
        }
      }
      __syncthreads();
      // exact online softmax update per head
      for (int h = tid; h < H; h += blockDim.x) {
        float mt = -INFINITY;
        for (int t = 0; t < kSimtRows; ++t) mt = fmaxf(mt, sc[h * kSimtRows + t]);
        const float mn = fmaxf(mref[h], mt);
        const float a = exp2f(mref[h] - mn);
        float ls = 0.f;
        for (int t = 0; t < kSimtRows; ++t) {
          const float pv = (t < nvalid) ? exp2f(sc[h * kSimtRows + t] - mn) : 0.f;
          pm[h * kSimtRows + t] = pv;
          ls += pv;
        }
        lsum[h] = lsum[h] * a + ls;
        mref[h] = mn;
        alph[h] = a;
      }
      __syncthreads();
      if (VARIANT_A) {
        for (int col = tid; col < d; col += blockDim.x) {
          const int h = col / d_h;
          float x = acc[col] * alph[h];
          for (int t = 0; t < kSimtRows; ++t) x = fmaf(pm[h * kSimtRows + t], to_f<KT>(vs[t * d + col]), x);
          acc[col] = x;
        }
      } else {
        for (int i = tid; i < H * d; i += blockDim.x) {
          const int h = i / d, col = i % d;
          float x = acc[i] * alph[h];
          for (int t = 0; t < kSimtRows; ++t) x = fmaf(pm[h * kSimtRows + t], to_f<KT>(ks[t * d + col]), x);
          acc[i] = x;
        }
      }
      __syncthreads();
    }
    const size_t slot = static_cast<size_t>(it.slot);
    for (int i = tid; i < nacc; i += blockDim.x) p.ws_U[slot * nacc + i] = acc[i];
    for (int h = tid; h < H; h += blockDim.x) {
      p.ws_m[slot * H + h] = mref[h];
      p.ws_l[slot * H + h] = lsum[h];
    }
    __syncthreads();  // the next segment reuses q, the accumulator and the softmax state
  }
}

// ---------------------------------------------------------------------------- append (ordering (a))
template <typename KT>
__global__ void append_kernel(const KT* __restrict__ k_new, KT* kcache, const int32_t* __restrict__ lens, int B,
                              int d, int64_t cap) {
  const int b = blockIdx.x;
  const int L = lens[b];
  if (L < 0 || static_cast<int64_t>(L) >= cap) return;  // reported by the split kernel's plan
  for (int i = threadIdx.x; i < d; i += blockDim.x)
    kcache[(static_cast<size_t>(b) * cap + L) * d + i] = k_new[static_cast<size_t>(b) * d + i];
}

// ---------------------------------------------------------------------------- row GEMM
// mode 0 (prompt phase): rows r < n of sequence b: in = X[b][r], out = cache[b][lens[b] + r];
//                         sequence skipped when lens[b] + n > cap.
// mode 1 (ordering (a)):  rows r < lens[b] + extra: in = cache[b][r], out = vbuf[b][r].
struct RowsGemmParams {
  const void* A;
  const void* W;
  void* Y;
  const int32_t* lens;
  int B, n, d, mode, extra;
  int64_t cap;
};

constexpr int kGemmBM = 32, kGemmBN = 64, kGemmBK = 32;

template <typename T>
__global__ void __launch_bounds__(256) rows_gemm_kernel(const RowsGemmParams p) {
  __shared__ float As[kGemmBM][kGemmBK + 1];
  __shared__ float Ws[kGemmBK][kGemmBN];
  const int b = blockIdx.z;
  const int L = p.lens[b];
  int nrows;
  if (p.mode == 0) {
    nrows = (L < 0 || static_cast<int64_t>(L) + p.n > p.cap) ? 0 : p.n;
  } else {
    const int64_t v = static_cast<int64_t>(L) + p.extra;
    nrows = (L < 0 || v > p.cap) ? 0 : static_cast<int>(v);
  }
  const int m0 = blockIdx.y * kGemmBM, n0 = blockIdx.x * kGemmBN;
  if (m0 >= nrows) return;
  const T* A = static_cast<const T*>(p.A);
  const T* W = static_cast<const T*>(p.W);
  T* Y = static_cast<T*>(p.Y);
  const size_t in_base = (p.mode == 0) ? static_cast<size_t>(b) * p.n : static_cast<size_t>(b) * p.cap;
  const size_t out_base = (p.mode == 0) ? static_cast<size_t>(b) * p.cap + L : static_cast<size_t>(b) * p.cap;
  const int tid = threadIdx.x;
  const int tr = tid / 16, tc = tid % 16;  // 2 rows x 4 cols per thread
  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  for (int k0 = 0; k0 < p.d; k0 += kGemmBK) {
    for (int i = tid; i < kGemmBM * kGemmBK; i += 256) {
      const int r = i / kGemmBK, c = i % kGemmBK;
      const int gr = m0 + r, gc = k0 + c;
      As[r][c] = (gr < nrows && gc < p.d) ? to_f<T>(A[(in_base + gr) * p.d + gc]) : 0.f;
    }
    for (int i = tid; i < kGemmBK * kGemmBN; i += 256) {
      const int r = i / kGemmBN, c = i % kGemmBN;
      const int gr = k0 + r, gc = n0 + c;
      Ws[r][c] = (gr < p.d && gc < p.d) ? to_f<T>(W[static_cast<size_t>(gr) * p.d + gc]) : 0.f;
    }
    __syncthreads();
    const int kend = min(kGemmBK, p.d - k0);
    for (int k = 0; k < kend; ++k) {
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = __fmaf_rn(As[tr * 2 + i][k], Ws[k][tc * 4 + j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int gr = m0 + tr * 2 + i;
    if (gr >= nrows) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gc = n0 + tc * 4 + j;
      if (gc < p.d) Y[(out_base + gr) * p.d + gc] = from_f<T>(acc[i][j]);
    }
  }
}

// ---------------------------------------------------------------------------- host
namespace {
SimtParams make_simt(const DecodeArgs& a, const SplitWorkspace& ws, bool variant_a) {
  SimtParams p;
  p.q = a.q;
  p.k_new = a.k_new;
  p.kcache = a.kcache;
  p.vbuf = ws.vbuf;
  p.lens = a.lens;
  p.status = a.status;
  p.ws_U = ws.U;
  p.ws_m = ws.m;
  p.ws_l = ws.l;
  p.ws_meta = ws.meta;
  p.B = a.B;
  p.d = a.d;
  p.H = a.H;
  p.cap = a.cap;
  const int app = a.k_new != nullptr ? 1 : 0;
  p.append = variant_a ? 0 : app;
  p.attend_add = app;
  p.n_slots = num_sms();
  p.min_rows = max(16, 8 * a.H);
  p.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(a.d / a.H));
  return p;
}

template <bool VA>
cudaError_t launch_simt(const DecodeArgs& a, const SplitWorkspace& ws, cudaStream_t st) {
  const SimtParams p = make_simt(a, ws, VA);
  const size_t smem = simt_smem_bytes(a.d, a.H, a.B, VA, a.dtype == SLIM_BF16 ? 2 : 4);
  if (smem > static_cast<size_t>(max_smem_optin())) return cudaErrorNotSupported;
  auto kern = (a.dtype == SLIM_BF16) ? decode_simt_kernel<__nv_bfloat16, VA> : decode_simt_kernel<float, VA>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<p.n_slots, 256, smem, st>>>(p);
  return cudaGetLastError();
}
}  // namespace

bool decode_b_simt_supported(int B, int d, int H) {
  return simt_smem_bytes(d, H, B, false, 2) <= static_cast<size_t>(max_smem_optin());
}

cudaError_t launch_decode_b_simt(const DecodeArgs& a, const SplitWorkspace& ws, cudaStream_t st, int* launches) {
  cudaError_t e = launch_simt<false>(a, ws, st);
  if (e == cudaSuccess && launches) ++*launches;
  return e;
}

cudaError_t launch_reduce_a(const DecodeArgs& a, const SplitWorkspace& ws, cudaStream_t st, int* launches);

bool decode_a_supported(int dtype, int B, int d, int H) {
  return simt_smem_bytes(d, H, B, true, dtype == SLIM_BF16 ? 2 : 4) <= static_cast<size_t>(max_smem_optin());
}

cudaError_t launch_rows_gemm(const void* A, const void* W, void* Y, const int32_t* lens, int rows_extra, int dtype,
                             int B, int d, int64_t cap, cudaStream_t st, int* launches) {
  RowsGemmParams p{A, W, Y, lens, B, 0, d, 1, rows_extra, cap};
  const dim3 grid((d + kGemmBN - 1) / kGemmBN, static_cast<unsigned>((cap + kGemmBM - 1) / kGemmBM), B);
  if (dtype == SLIM_BF16) rows_gemm_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(p);
  else rows_gemm_kernel<float><<<grid, 256, 0, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess && launches) ++*launches;
  return e;
}

cudaError_t launch_prefill_simt(const void* X, const void* W, void* kcache, const int32_t* lens, int dtype, int B,
                                int n, int d, int64_t cap, cudaStream_t st, int* launches) {
  RowsGemmParams p{X, W, kcache, lens, B, n, d, 0, 0, cap};
  const dim3 grid((d + kGemmBN - 1) / kGemmBN, (n + kGemmBM - 1) / kGemmBM, B);
  if (dtype == SLIM_BF16) rows_gemm_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(p);
  else rows_gemm_kernel<float><<<grid, 256, 0, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess && launches) ++*launches;
  return e;
}

cudaError_t launch_decode_a(const DecodeArgs& a, const SplitWorkspace& ws, cudaStream_t st, int* launches) {
  const int app = a.k_new != nullptr ? 1 : 0;
  cudaError_t e = cudaSuccess;
  if (app) {
    if (a.dtype == SLIM_BF16)
      append_kernel<__nv_bfloat16><<<a.B, 128, 0, st>>>(static_cast<const __nv_bfloat16*>(a.k_new),
                                                          static_cast<__nv_bfloat16*>(a.kcache), a.lens, a.B, a.d,
                                                          a.cap);
    else
      append_kernel<float><<<a.B, 128, 0, st>>>(static_cast<const float*>(a.k_new), static_cast<float*>(a.kcache),
                                                a.lens, a.B, a.d, a.cap);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (launches) ++*launches;
  }
  if (decode_a_tc_supported(a.dtype, a.B, a.d, a.H)) return launch_decode_a_tc(a, ws, st, launches);
  e = launch_rows_gemm_any(a.kcache, a.w_kv, ws.vbuf, a.lens, app, a.dtype, a.B, a.d, a.cap, a.status, st,
                           launches);
  if (e != cudaSuccess) return e;
  e = launch_simt<true>(a, ws, st);
  if (e != cudaSuccess) return e;
  if (launches) ++*launches;
  return launch_reduce_a(a, ws, st, launches);
}

}  // namespace slim
