// Row GEMM Y = A·W on tcgen05 tensor cores (bf16 in, fp32 accumulation, bf16 out).
//
// Two uses (Slim Attention article, section "K-Cache is All You Need"):
//   * prompt phase: K = X·W_K for n new tokens of every sequence, written to
//     cache rows lens[b] .. lens[b]+n-1 (V is not computed);
//   * V = K·W_KV for the cached rows of every sequence into a V buffer with the
//     cache's layout (the prompt phase's attention output, ordering (a)).
// Persistent CTAs (one per SM) walk the 128-row x 256-column output tiles of
// all sequences, column tiles innermost so that consecutive tiles share their
// rows in L2. Warp 0 issues TMA loads (A: 128 rows x 64 columns, K-major,
// 128-byte swizzle; W: 64 rows x 256 columns as four MN-major 64-column
// blocks) into a 4-stage ring; warp 1 issues tcgen05.mma M=128 N=256 K=16
// into one of two 256-column TMEM accumulators; warps 2..5 convert a finished
// accumulator to bf16 and store it while the next tile's main loop runs.
#include <cuda_bf16.h>

#include <algorithm>

#include "ptx.cuh"

namespace slim {

namespace {

constexpr int kBM = 128, kBN = 256, kBK = 64, kStages = 4;
constexpr int kGemmThreads = 192;
constexpr uint32_t kAStage = kBM * kBK * 2;  // 16 KB
constexpr uint32_t kBStage = kBK * kBN * 2;  // 32 KB
constexpr uint32_t kGemmSmem = kStages * (kAStage + kBStage) + 1024 + 256;

struct GemmParams {
  __nv_bfloat16* Y;
  const int32_t* lens;
  int B, n, d, mode, extra;  // mode 0: prompt rows of X; mode 1: attended cache rows
  int64_t cap;
  int64_t a_rows_per_seq;    // rows per sequence in the A tensor map (n or cap)
  int mtiles;                // row tiles per sequence in the tile grid
};

__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap wmap,
                   const GemmParams p, int32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* as = smem;
  uint8_t* bs = smem + kStages * kAStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * (kAStage + kBStage));
  uint64_t* empty = full + kStages;
  uint64_t* accfull = empty + kStages;  // [2]
  uint64_t* accempty = accfull + 2;     // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accempty + 2);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = p.d / kBN, nk = p.d / kBK;
  const int n_tiles = p.B * p.mtiles * ntiles;

  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&amap);
    tma_prefetch_desc(&wmap);
  } else if (warp == 1) {
    if (lane == 0) {
      for (int s = 0; s < kStages; ++s) {
        mbar_init(&full[s], 1);
        mbar_init(&empty[s], 1);
      }
      for (int a = 0; a < 2; ++a) {
        mbar_init(&accfull[a], 1);
        mbar_init(&accempty[a], 4);
      }
      fence_barrier_init();
    }
    __syncwarp();
    tmem_alloc(tmem_slot, 2 * kBN);
    tmem_relinquish();
  }
  pdl_wait_primary();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // rows of tile tau to produce (0: nothing) and where they go
  auto tile_of = [&](int tau, int& b, int& m0, int& n0, int& nrows, int64_t& out_row0) {
    const int nt = tau % ntiles, rest = tau / ntiles;
    const int mt = rest % p.mtiles;
    b = rest / p.mtiles;
    m0 = mt * kBM;
    n0 = nt * kBN;
    const int L = __ldg(p.lens + b);
    if (p.mode == 0) {
      nrows = (L < 0 || static_cast<int64_t>(L) + p.n > p.cap) ? 0 : p.n;
      out_row0 = static_cast<int64_t>(b) * p.cap + L;
    } else {
      const int64_t v = static_cast<int64_t>(L) + p.extra;
      nrows = (L < 0 || v > p.cap) ? 0 : static_cast<int>(v);
      out_row0 = static_cast<int64_t>(b) * p.cap;
    }
    return m0 < nrows;
  };

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_a = l2_policy_evict_first();
      const uint64_t pol_w = l2_policy_evict_last();
      int g = 0;
      bool ok = true;
      for (int tau = blockIdx.x; tau < n_tiles && ok; tau += gridDim.x) {
        int b, m0, n0, nrows;
        int64_t orow;
        if (!tile_of(tau, b, m0, n0, nrows, orow)) continue;
        const int a_row = static_cast<int>(static_cast<int64_t>(b) * p.a_rows_per_seq + m0);
        for (int k = 0; k < nk; ++k, ++g) {
          const int s = g % kStages;
          const uint32_t ph = static_cast<uint32_t>(g / kStages) & 1u;
          if (g >= kStages && !mbar_wait(&empty[s], ph ^ 1u, status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], kAStage + kBStage);
          tma_load_2d(as + s * kAStage, &amap, k * kBK, a_row, &full[s], pol_a);
          tma_load_3d(bs + s * kBStage, &wmap, 0, k * kBK, n0 / 64, &full[s], pol_w);
        }
      }
      for (int t = max(0, g - kStages); t < g; ++t)  // every issued copy lands before exit
        mbar_wait(&full[t % kStages], static_cast<uint32_t>(t / kStages) & 1u, status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kBM, kBN, 0u, 1u);
      const uint32_t abase = smem_u32(as), bbase = smem_u32(bs);
      int g = 0, i = 0;
      bool ok = true;
      for (int tau = blockIdx.x; tau < n_tiles && ok; tau += gridDim.x) {
        int b, m0, n0, nrows;
        int64_t orow;
        if (!tile_of(tau, b, m0, n0, nrows, orow)) continue;
        const int ab = i & 1;
        // the epilogue of tile i - 2 must have read this accumulator
        if (i >= 2 && !mbar_wait(&accempty[ab], static_cast<uint32_t>((i - 2) >> 1) & 1u, status)) break;
        tc_fence_after();
        const uint32_t acc = tmem + static_cast<uint32_t>(ab * kBN);
        for (int k = 0; k < nk; ++k, ++g) {
          const int s = g % kStages;
          const uint32_t ph = static_cast<uint32_t>(g / kStages) & 1u;
          if (!mbar_wait(&full[s], ph, status)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            // A: K-major, 128-byte swizzle, 8-row groups 1024 B apart; a 16-column step is 32 B.
            const uint64_t ad = smem_desc(abase + s * kAStage + kk * 32, 16, 1024, kLayoutSW128);
            // W: MN-major, 64-column blocks 64 rows x 128 B (8 KB) apart, 8-row groups 1024 B apart.
            const uint64_t bd = smem_desc(bbase + s * kBStage + kk * 16 * 128, kBK * 128, 1024, kLayoutSW128);
            umma_f16(acc, ad, bd, idesc, (k > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty[s]);
        }
        umma_commit(&accfull[ab]);  // also after a failed chunk: covers every MMA issued so far
        ++i;
      }
      if (i > 0) mbar_wait(&accfull[(i - 1) & 1], static_cast<uint32_t>((i - 1) >> 1) & 1u, status);
    }
  } else {
    // epilogue: TMEM lane = tile row, columns = output columns
    const int quarter = warp & 3;
    int i = 0;
    for (int tau = blockIdx.x; tau < n_tiles; tau += gridDim.x) {
      int b, m0, n0, nrows;
      int64_t orow;
      if (!tile_of(tau, b, m0, n0, nrows, orow)) continue;
      const int ab = i & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&accfull[ab], static_cast<uint32_t>(i >> 1) & 1u, status))) break;
      tc_fence_after();
      const int r = m0 + quarter * 32 + lane;
      __nv_bfloat16* dst = p.Y + (orow + r) * p.d + n0;
      const uint32_t tacc = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(ab * kBN);
      for (int c = 0; c < kBN; c += 32) {
        float v[2][16];
        tmem_ld16(tacc + c, v[0]);
        tmem_ld16(tacc + c + 16, v[1]);
        tmem_wait_ld();
        if (r < nrows) {
#pragma unroll
          for (int hx = 0; hx < 2; ++hx) {
            uint4 o0, o1;
            o0.x = pack_bf16x2(v[hx][0], v[hx][1]);
            o0.y = pack_bf16x2(v[hx][2], v[hx][3]);
            o0.z = pack_bf16x2(v[hx][4], v[hx][5]);
            o0.w = pack_bf16x2(v[hx][6], v[hx][7]);
            o1.x = pack_bf16x2(v[hx][8], v[hx][9]);
            o1.y = pack_bf16x2(v[hx][10], v[hx][11]);
            o1.z = pack_bf16x2(v[hx][12], v[hx][13]);
            o1.w = pack_bf16x2(v[hx][14], v[hx][15]);
            *reinterpret_cast<uint4*>(dst + c + 16 * hx) = o0;
            *reinterpret_cast<uint4*>(dst + c + 16 * hx + 8) = o1;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&accempty[ab]);
      ++i;
    }
  }
  __syncwarp();  // lanes 1..31 of warps 0 and 1 skipped the lane-0 loops: reconverge before the CTA barrier
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * kBN);
  }
}

// W [d rows][d cols] bf16 viewed as {64 columns, d rows, d/64 column blocks}; box 64 x 64 x 4.
bool encode_wmap(CUtensorMap* map, const void* W, int d) {
  return encode_tmap_3d_bf16(map, W, 64, static_cast<uint64_t>(d), static_cast<uint64_t>(d / 64),
                             static_cast<uint64_t>(d) * 2u, 128u, 64, kBK, kBN / 64);
}

cudaError_t launch_gemm(const void* A, uint64_t a_rows_total, int64_t a_rows_per_seq, const void* W, void* Y,
                        const int32_t* lens, int B, int n, int d, int64_t cap, int mode, int extra, int grid_rows,
                        int32_t* status, cudaStream_t st, int* launches) {
  CUtensorMap amap, wmap;
  if (!encode_tmap_2d_bf16(&amap, A, static_cast<uint64_t>(d), a_rows_total, static_cast<uint64_t>(d) * 2u, kBK,
                           kBM, true) ||
      !encode_wmap(&wmap, W, d))
    return cudaErrorInvalidValue;
  const int mtiles = (grid_rows + kBM - 1) / kBM;
  GemmParams p{static_cast<__nv_bfloat16*>(Y), lens, B, n, d, mode, extra, cap, a_rows_per_seq, mtiles};
  cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmem);
  if (e != cudaSuccess) return e;
  const long long tiles = static_cast<long long>(B) * mtiles * (d / kBN);
  const unsigned grid = static_cast<unsigned>(std::min<long long>(tiles, num_sms()));
  gemm_tc_kernel<<<grid, kGemmThreads, kGemmSmem, st>>>(amap, wmap, p, status);
  e = cudaGetLastError();
  if (e == cudaSuccess && launches) ++*launches;
  return e;
}

}  // namespace

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

bool gemm_tc_supported(int d) { return d >= kBN && d % kBN == 0; }

cudaError_t launch_prefill_tc(const void* X, const void* W, void* kcache, const int32_t* lens, int B, int n, int d,
                              int64_t cap, int32_t* status, cudaStream_t st, int* launches) {
  if (!gemm_tc_supported(d)) return cudaErrorNotSupported;
  return launch_gemm(X, static_cast<uint64_t>(B) * n, n, W, kcache, lens, B, n, d, cap, 0, 0, n, status, st,
                     launches);
}

cudaError_t launch_rows_gemm_tc(const void* A, const void* W, void* Y, const int32_t* lens, int rows_extra, int B,
                                int d, int64_t cap, int32_t* status, cudaStream_t st, int* launches) {
  if (!gemm_tc_supported(d)) return cudaErrorNotSupported;
  return launch_gemm(A, static_cast<uint64_t>(B) * cap, cap, W, Y, lens, B, 0, d, cap, 1, rows_extra,
                     static_cast<int>(cap), status, st, launches);
}

}  // namespace slim
