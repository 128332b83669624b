// Merge of the split-T partials and the W_KV projection.
//
// Ordering (b) (Slim Attention article, section "K-Cache is All You Need",
// second generation-phase option, with W_KV = W_K^(-1)·W_V): for sequence b
// and head h, the partials (m_c, l_c, U_c) of the sequence's segments combine
// by the log-sum-exp rule into
//     ū = Σ_c 2^(m_c - M) U_c / Σ_c 2^(m_c - M) l_c,   M = max_c m_c,
// and the head output is  o[b, h-cols] = ū · W_KV[:, h-cols].
//
// Three kernels, chosen by shape (launch_reduce_b):
//   * merge_lean_kernel  one CTA per (head, sequence): d_h = 64, d <= 1280 and
//     B·H CTAs in one wave; the head slice of W_KV is held whole in shared memory.
//   * merge_proj_kernel  bf16 W_KV with d_h = 64 or 128, any batch: one CTA per
//     (head, block of d rows), all CTAs in one wave, clusters along the blocks.
//     The partial rows are read with many loads in flight per thread and summed
//     into a bf16 high/low tcgen05 operand; W_KV streams through a ring of TMA
//     tiles and the projection runs on tcgen05 with a TMEM accumulator; the
//     blocks' products are summed in a fixed order through distributed shared
//     memory.
//   * merge_b_kernel     the same decomposition on the CUDA cores, for fp32
//     W_KV (and bf16 shapes the other two do not take).
// Each is a programmatic dependent of the split kernel: what does not depend
// on the split's results (barriers, the first W_KV tiles) happens before the
// wait.
//
// Ordering (a) needs only the merge (its partials are already softmax·V).
#include <cuda_bf16.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>
#include <type_traits>
#include <utility>

#include "ptx.cuh"

namespace slim {

struct MergeBParams {
  const float* U;
  const float* m;
  const float* l;
  const int32_t* meta;
  float* out;
  int32_t* lens;
  int32_t* status;
  int B, d, H, ndb, max_items;
  int b_begin, nb;  // sequences of this launch
};

constexpr int kMergeThreads = 256;
constexpr int kMergeWarps = kMergeThreads / 32;
constexpr int kMergeMaxSeqs = 128;  // sequences per launch (MMA rows)
constexpr int kMergeRound = 8;      // 16-byte loads in flight per thread and round

struct MergeSmem {
  uint32_t w, ub, ubs, wts, ls, soff, part, recv, per, bars, total;
};
__host__ __device__ inline uint32_t up_to(uint32_t x, uint32_t a) { return (x + a - 1u) / a * a; }
__host__ __device__ inline MergeSmem merge_smem_layout(int DB, int d_h, int esz, int nb, int ndb, int ncap) {
  MergeSmem s;
  uint32_t o = 0;
  s.w = o;  // W_KV block [DB rows][d_h]: 64-column 128-byte-swizzled boxes (MMA) or dense rows
  o += up_to(static_cast<uint32_t>(DB) * d_h * esz, 1024u);
  s.ubs = static_cast<uint32_t>(DB) + 8u;  // row stride of ū (floats), padded against bank conflicts
  s.ub = o;
  o += up_to(static_cast<uint32_t>(nb), 16u) * s.ubs * 4u;
  s.wts = o;
  o += up_to(static_cast<uint32_t>(ncap), 4u) * 4u;
  s.ls = o;
  o += up_to(static_cast<uint32_t>(ncap), 4u) * 4u;
  s.soff = o;
  o += up_to(static_cast<uint32_t>(nb) + 1u, 4u) * 4u;
  s.part = o;  // this CTA's product [nb][d_h]
  o += static_cast<uint32_t>(nb) * d_h * 4u;
  s.per = (static_cast<uint32_t>(nb) * d_h + ndb - 1u) / ndb;  // output elements owned per CTA
  s.recv = o;  // products pushed by the NDB CTAs of the cluster: [NDB][per]
  o += static_cast<uint32_t>(ndb) * s.per * 4u;
  o = up_to(o, 8u);
  s.bars = o;
  o += 16u;
  s.total = o + 1024u;  // slack to align the base to 1024 bytes
  return s;
}

template <typename WT>
__global__ void __launch_bounds__(kMergeThreads, 2)
    merge_b_kernel(const __grid_constant__ CUtensorMap wmap, const MergeBParams p) {
  extern __shared__ uint8_t msm_raw[];
  uint8_t* msm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(msm_raw) + 1023) & ~uintptr_t(1023));
  const int h = blockIdx.x, r = blockIdx.y;
  const int d_h = p.d / p.H, DB = p.d / p.ndb, c0 = r * DB;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nb = p.nb, b0 = p.b_begin, Bp = (nb + 15) & ~15;
  const MergeSmem L = merge_smem_layout(DB, d_h, static_cast<int>(sizeof(WT)), nb, p.ndb, p.max_items);
  float* ub = reinterpret_cast<float*>(msm + L.ub);
  float* wts = reinterpret_cast<float*>(msm + L.wts);  // m of every item, then its merge weight
  float* ls = reinterpret_cast<float*>(msm + L.ls);
  int* s_off = reinterpret_cast<int*>(msm + L.soff);  // items of sequence b0 + i start at s_off[i]
  float* part = reinterpret_cast<float*>(msm + L.part);
  float* recv = reinterpret_cast<float*>(msm + L.recv);
  uint64_t* wbar = reinterpret_cast<uint64_t*>(msm + L.bars);
  const int ubs = static_cast<int>(L.ubs), per = static_cast<int>(L.per);

  // ---- before the split kernel's results exist: barrier, W_KV block, zeroed ū
  if (tid == 0) {
    mbar_init(wbar, 1);
    fence_barrier_init();
    tma_prefetch_desc(&wmap);
    const int yrows = min(DB, 256);
    mbar_arrive_expect_tx(wbar, static_cast<uint32_t>(DB) * d_h * sizeof(WT));
    for (int y = 0; y < DB; y += yrows)
      tma_load_2d(msm + L.w + static_cast<size_t>(y) * d_h * sizeof(WT), &wmap, h * d_h, c0 + y, wbar,
                  l2_policy_evict_last());
  }
  for (int i = tid; i < Bp * ubs; i += kMergeThreads) ub[i] = 0.f;
  if (p.ndb > 1) cluster_arrive_relaxed();
  pdl_wait_primary();
  pdl_launch_dependents();

  // ---- every load at once: this thread's U slices, then the work list and m, l
  const int it0 = b0 == 0 ? 0 : __ldcg(p.meta + 1 + b0);
  const int ncap = p.max_items - it0;
  // Thread (cg, ig) takes columns 4cg.. of a contiguous run of slots (runs of one sequence
  // then add up in registers), balanced over the slots the split kernel produced.
  const int C4 = DB / 4, IG = kMergeThreads / C4;
  const int cg = tid % C4, ig = tid < IG * C4 ? tid / C4 : IG;
  const int n_real = min(ncap, __ldcg(p.meta + 1 + b0 + nb) - it0);  // slots of this launch's sequences
  const int ipt = (n_real + IG - 1) / IG;
  const int i_beg = ig * ipt;
  const int i_end = ig < IG ? min(n_real, i_beg + ipt) : i_beg;
  const float4* ubase = reinterpret_cast<const float4*>(p.U + (static_cast<size_t>(it0) * p.H + h) * p.d + c0) + cg;
  const size_t istride = static_cast<size_t>(p.H) * p.d / 4;  // float4 stride between items
  const int nrounds = (ipt + kMergeRound - 1) / kMergeRound;
  float4 bufA[kMergeRound], bufB[kMergeRound];
  auto load_round = [&](float4 (&buf)[kMergeRound], int rr) {
#pragma unroll
    for (int u = 0; u < kMergeRound; ++u) {
      const int i = i_beg + rr * kMergeRound + u;
      buf[u] = i < i_end ? __ldcg(ubase + static_cast<size_t>(i) * istride) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  load_round(bufA, 0);
  if (nrounds > 1) load_round(bufB, 1);
  for (int i = tid; i <= nb; i += kMergeThreads) s_off[i] = __ldcg(p.meta + 1 + b0 + i) - it0;
  for (int i = tid; i < ncap; i += kMergeThreads) {
    wts[i] = __ldcg(p.m + static_cast<size_t>(it0 + i) * p.H + h);
    ls[i] = __ldcg(p.l + static_cast<size_t>(it0 + i) * p.H + h);
  }
  if (h == 0 && r == 0)
    for (int b = b0 + tid; b < b0 + nb; b += kMergeThreads)
      if (__ldcg(p.meta + 2 + p.B + b) & kSeqAppend) p.lens[b] += 1;
  __syncthreads();

  // ---- merge weights 2^(m_c - M) / Σ_c' 2^(m_c' - M) l_c', one warp per sequence
  for (int bl = warp; bl < nb; bl += kMergeWarps) {
    const int lo = s_off[bl], hi = s_off[bl + 1];
    float M = -INFINITY;
    for (int c = lo + lane; c < hi; c += 32) M = fmaxf(M, wts[c]);
    M = warp_max(M);
    float S = 0.f;
    for (int c = lo + lane; c < hi; c += 32) S += exp2f(wts[c] - M) * ls[c];
    S = warp_sum(S);
    const float inv = S > 0.f ? 1.f / S : 0.f;
    for (int c = lo + lane; c < hi; c += 32) wts[c] = exp2f(wts[c] - M) * inv;
  }
  __syncthreads();

  // ---- ū[b, block] = Σ_c w_c U_c[block]: runs of one sequence add up in registers
  if (i_beg < i_end) {
    int bcur = 0;
    while (bcur < nb && s_off[bcur + 1] <= i_beg) ++bcur;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    auto flush = [&]() {
      if (bcur < nb) {
        float* dst = ub + bcur * ubs + 4 * cg;
        red_shared_add(dst, acc.x);
        red_shared_add(dst + 1, acc.y);
        red_shared_add(dst + 2, acc.z);
        red_shared_add(dst + 3, acc.w);
      }
      acc = make_float4(0.f, 0.f, 0.f, 0.f);
    };
    auto consume = [&](const float4 (&buf)[kMergeRound], int rr) {
#pragma unroll
      for (int u = 0; u < kMergeRound; ++u) {
        const int i = i_beg + rr * kMergeRound + u;
        if (i >= i_end) break;
        while (bcur < nb && i >= s_off[bcur + 1]) {
          flush();
          ++bcur;
        }
        if (bcur >= nb) break;
        const float w = wts[i];
        acc.x = fmaf(w, buf[u].x, acc.x);
        acc.y = fmaf(w, buf[u].y, acc.y);
        acc.z = fmaf(w, buf[u].z, acc.z);
        acc.w = fmaf(w, buf[u].w, acc.w);
      }
    };
    for (int rr = 0; rr < nrounds; rr += 2) {
      consume(bufA, rr);
      if (rr + 2 < nrounds) load_round(bufA, rr + 2);
      if (rr + 1 < nrounds) {
        consume(bufB, rr + 1);
        if (rr + 3 < nrounds) load_round(bufB, rr + 3);
      }
    }
    flush();
  }
  const bool ok = __syncthreads_and(mbar_wait(wbar, 0u, p.status));
  // after a wait that gave up, the block copy may still be landing in this CTA's shared memory:
  // one more bounded wait keeps the CTA alive until it has (copies always complete)
  if (!ok && tid == 0) mbar_wait(wbar, 0u, p.status);

  // ---- this CTA's product o_r[b, :] = ū[b, block] · W_KV[block, h-cols]
  if (ok) {
    // FMAs: thread -> (sequence, 4 columns, one of S interleaved row subsets of the block),
    // the S partial sums (adjacent lanes) added with shuffles
    const WT* wsm = reinterpret_cast<const WT*>(msm + L.w);
    const int pairs = nb * (d_h / 4);
    int S = 1;
    while (S < 32 && pairs * S * 2 <= kMergeThreads) S *= 2;
    for (int q0 = 0; q0 < pairs * S; q0 += kMergeThreads) {
      const int q = q0 + tid;
      const int pr = q / S, cs = q % S;
      const int bl = pr / (d_h / 4), j = 4 * (pr - bl * (d_h / 4));
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
      if (pr < pairs) {
        for (int c = cs; c < DB; c += S) {
          const float u = ub[bl * ubs + c];
          float w[4];
          const WT* wr = wsm + static_cast<size_t>(c) * d_h + j;
#pragma unroll
          for (int v = 0; v < 4; ++v) w[v] = static_cast<float>(wr[v]);
          a.x = fmaf(u, w[0], a.x);
          a.y = fmaf(u, w[1], a.y);
          a.z = fmaf(u, w[2], a.z);
          a.w = fmaf(u, w[3], a.w);
        }
      }
      for (int o = 1; o < S; o <<= 1) {
        a.x += __shfl_xor_sync(0xffffffffu, a.x, o);
        a.y += __shfl_xor_sync(0xffffffffu, a.y, o);
        a.z += __shfl_xor_sync(0xffffffffu, a.z, o);
        a.w += __shfl_xor_sync(0xffffffffu, a.w, o);
      }
      if (pr < pairs && cs == 0) *reinterpret_cast<float4*>(part + bl * d_h + j) = a;
    }
  }
  __syncthreads();

  // ---- sum the NDB products: push each element to its owner CTA, then add in a fixed order
  const int n_out = nb * d_h;
  if (p.ndb == 1) {
    for (int e = tid; e < n_out; e += kMergeThreads)
      p.out[static_cast<size_t>(b0 + e / d_h) * p.d + h * d_h + e % d_h] = ok ? part[e] : 0.f;
    return;
  }
  cluster_wait();  // every CTA of the cluster is running
  const uint32_t recv_base = smem_u32(recv);
  for (int e = tid; e < n_out; e += kMergeThreads)
    st_cluster_f32(mapa_shared(recv_base + 4u * static_cast<uint32_t>(r * per + e / p.ndb), e % p.ndb),
                   ok ? part[e] : 0.f);
  cluster_sync();  // pushes visible; nobody touches a peer's shared memory after this
  for (int s = tid; s < per; s += kMergeThreads) {
    const int e = s * p.ndb + r;
    if (e >= n_out) break;
    float a = 0.f;
    for (int q = 0; q < p.ndb; ++q) a += recv[q * per + s];
    p.out[static_cast<size_t>(b0 + e / d_h) * p.d + h * d_h + e % d_h] = a;
  }
}

// ---------------------------------------------------------------------------- one-sequence merge
// The same merge and projection for shapes whose head slice of W_KV fits in shared memory
// (d_h = 64, d <= 1280) and whose B x H CTAs fit in one wave: CTA (h, b) owns head h of
// sequence b entirely, so no cluster reduction follows the projection.
//   * Before the split kernel's results are awaited: W_KV[:, h-cols] (d rows x 128 bytes,
//     128-byte swizzled) by TMA.
//   * The item range of sequence b, then in one round trip the items' m and l and their U rows
//     of head h (one bulk copy of d floats per item, completing on an mbarrier).
//   * Every thread holds the columns tid + 256 i of ū = Σ_c 2^(m_c - M) U_c / Σ_c 2^(m_c - M) l_c
//     and multiplies them by the matching W_KV rows (conflict-free swizzled 16-byte reads);
//     a butterfly over the warp leaves two of the 64 outputs per lane, and 64 threads add the
//     eight warps' sums.
struct MergeLeanParams {
  const float* U;
  const float* m;
  const float* l;
  const int32_t* meta;
  float* out;
  int32_t* lens;
  int32_t* status;
  int B, d, H, max_items;
  int cap_items;  // U rows staged per round
};

constexpr int kLeanThreads = 256;
constexpr int kLeanDh = 64;
constexpr int kLeanMaxCols = 1280;
constexpr int kLeanCols = kLeanMaxCols / kLeanThreads;  // columns of ū per thread
constexpr int kLeanWBlk = kLeanThreads / 32;              // items per sequence <= 32 * kLeanWBlk

struct LeanSmem {
  uint32_t w, u, wt, red, bars, total;
};
__host__ __device__ inline LeanSmem lean_smem_layout(int d, int cap_items, int max_items) {
  LeanSmem s;
  uint32_t o = 0;
  s.w = o;  // [d rows][64 bf16], 128-byte swizzle (1024-byte aligned base)
  o += up_to(static_cast<uint32_t>(d) * kLeanDh * 2u, 1024u);
  s.u = o;  // [cap_items][d] fp32
  o += static_cast<uint32_t>(cap_items) * d * 4u;
  s.wt = o;  // merge weight of every item of the sequence
  o += up_to(static_cast<uint32_t>(max_items) * 4u, 16u);
  s.red = o;  // [8 warps][64]
  o += (kLeanThreads / 32) * kLeanDh * 4u;
  s.bars = o;
  o += 32u;
  s.total = o + 1024u;  // slack to align the base to 1024 bytes
  return s;
}

// Warp 0: U rows of head h of items lo + r0 .. (at most cap) into shared memory, one bulk copy
// per lane, completing on ubar.
__device__ __forceinline__ void lean_stage(float* us, const float* U, int lo, int r0, int n, int cap, int H, int h,
                                           int d, uint64_t* ubar, int lane) {
  const int nr = min(n - r0, cap);
  const uint32_t row_bytes = static_cast<uint32_t>(d) * 4u;
  if (lane == 0) mbar_arrive_expect_tx(ubar, static_cast<uint32_t>(nr) * row_bytes);
  __syncwarp();
  for (int c = lane; c < nr; c += 32)
    bulk_load_g2s(us + static_cast<size_t>(c) * d, U + (static_cast<size_t>(lo + r0 + c) * H + h) * d, row_bytes,
                  ubar);
}

__global__ void __launch_bounds__(kLeanThreads, 1)
    merge_lean_kernel(const __grid_constant__ CUtensorMap wmap, const MergeLeanParams p) {
  extern __shared__ uint8_t lsm_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(lsm_raw) + 1023) & ~uintptr_t(1023));
  const LeanSmem L = lean_smem_layout(p.d, p.cap_items, p.max_items);
  const int h = blockIdx.x, b = blockIdx.y, d = p.d;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float* us = reinterpret_cast<float*>(sm + L.u);
  float* red = reinterpret_cast<float*>(sm + L.red);
  float* ws_ = reinterpret_cast<float*>(sm + L.wt);
  uint64_t* wbar = reinterpret_cast<uint64_t*>(sm + L.bars);
  uint64_t* ubar = wbar + 1;
  int* rng = reinterpret_cast<int*>(wbar + 2);

  if (tid == 0) {
    mbar_init(wbar, 1);
    mbar_init(ubar, 1);
    fence_barrier_init();
    tma_prefetch_desc(&wmap);
    mbar_arrive_expect_tx(wbar, static_cast<uint32_t>(d) * kLeanDh * 2u);
    for (int y = 0; y < d; y += 256)
      tma_load_2d(sm + L.w + static_cast<size_t>(y) * 128, &wmap, h * kLeanDh, y, wbar, l2_policy_evict_last());
  }
  __syncthreads();
  pdl_wait_primary();
  pdl_launch_dependents();

  if (tid < 2) rng[tid] = __ldcg(p.meta + 1 + b + tid);
  if (h == 0 && tid == 32 && (__ldcg(p.meta + 2 + p.B + b) & kSeqAppend)) p.lens[b] += 1;
  __syncthreads();
  const int lo = rng[0], n = rng[1] - lo;
  if (warp == 0 && n > 0) lean_stage(us, p.U, lo, 0, n, p.cap_items, p.H, h, d, ubar, lane);

  // merge weights 2^(m_c - M) / Σ_c' 2^(m_c' - M) l_c': every warp loads every item's m and l at
  // once (lane c % 32 of block c / 32) and finds M and the sum itself, so no barrier separates
  // them; warp j writes the weights of block j, published by the barrier of the first U wait
  const float* mh = p.m + static_cast<size_t>(lo) * p.H + h;
  const float* lh = p.l + static_cast<size_t>(lo) * p.H + h;
  float mv[kLeanWBlk], lv[kLeanWBlk];
#pragma unroll
  for (int j = 0; j < kLeanWBlk; ++j) {
    const int c = lane + 32 * j;
    mv[j] = c < n ? mh[static_cast<size_t>(c) * p.H] : -INFINITY;
    lv[j] = c < n ? lh[static_cast<size_t>(c) * p.H] : 0.f;
  }
  float M = mv[0];
#pragma unroll
  for (int j = 1; j < kLeanWBlk; ++j) M = fmaxf(M, mv[j]);
  M = warp_max(M);
  float S = 0.f;
#pragma unroll
  for (int j = 0; j < kLeanWBlk; ++j) {
    mv[j] = lane + 32 * j < n ? exp2f(mv[j] - M) : 0.f;
    S = fmaf(mv[j], lv[j], S);
  }
  S = warp_sum(S);
  const float inv = S > 0.f ? 1.f / S : 0.f;
#pragma unroll
  for (int j = 0; j < kLeanWBlk; ++j)
    if (warp == j && lane + 32 * j < n) ws_[lane + 32 * j] = mv[j] * inv;

  float ub[kLeanCols];
#pragma unroll
  for (int i = 0; i < kLeanCols; ++i) ub[i] = 0.f;
  bool ok = true;
  uint32_t ph = 0;
  for (int r0 = 0; r0 < n; r0 += p.cap_items, ph ^= 1u) {
    ok = __syncthreads_and(mbar_wait(ubar, ph, p.status));
    if (!ok) {
      if (tid == 0) mbar_wait(ubar, ph, p.status);  // drain the staged copies before leaving
      break;
    }
    const int nr = min(n - r0, p.cap_items);
    for (int c = 0; c < nr; ++c) {
      const float w = ws_[r0 + c];
      const float* row = us + static_cast<size_t>(c) * d;
#pragma unroll
      for (int i = 0; i < kLeanCols; ++i) {
        const int col = tid + kLeanThreads * i;
        if (col < d) ub[i] = fmaf(w, row[col], ub[i]);
      }
    }
    if (r0 + p.cap_items < n) {
      __syncthreads();  // every thread is done with the staged rows
      if (warp == 0) lean_stage(us, p.U, lo, r0 + p.cap_items, n, p.cap_items, p.H, h, d, ubar, lane);
    }
  }
  const bool w_ok = __syncthreads_and(mbar_wait(wbar, 0u, p.status));
  if (!w_ok && tid == 0) mbar_wait(wbar, 0u, p.status);  // the W_KV copy must land before exit
  ok = ok && w_ok;

  // o[j] = Σ_rows ū[row] W[row][j]: this thread's rows, all 64 outputs
  float acc[kLeanDh];
#pragma unroll
  for (int j = 0; j < kLeanDh; ++j) acc[j] = 0.f;
  const uint32_t wbase = smem_u32(sm + L.w);
#pragma unroll
  for (int i = 0; i < kLeanCols; ++i) {
    const int row = tid + kLeanThreads * i;
    if (row < d) {
      const float u = ub[i];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        uint4 v;
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                     : "r"(wbase + static_cast<uint32_t>(row) * 128u + ((static_cast<uint32_t>(k ^ (row & 7))) << 4)));
        acc[8 * k + 0] = fmaf(u, bf16lo(v.x), acc[8 * k + 0]);
        acc[8 * k + 1] = fmaf(u, bf16hi(v.x), acc[8 * k + 1]);
        acc[8 * k + 2] = fmaf(u, bf16lo(v.y), acc[8 * k + 2]);
        acc[8 * k + 3] = fmaf(u, bf16hi(v.y), acc[8 * k + 3]);
        acc[8 * k + 4] = fmaf(u, bf16lo(v.z), acc[8 * k + 4]);
        acc[8 * k + 5] = fmaf(u, bf16hi(v.z), acc[8 * k + 5]);
        acc[8 * k + 6] = fmaf(u, bf16lo(v.w), acc[8 * k + 6]);
        acc[8 * k + 7] = fmaf(u, bf16hi(v.w), acc[8 * k + 7]);
      }
    }
  }
  // butterfly reduce-scatter over the warp: after the stage with offset o a lane keeps the half
  // of its values selected by lane bit o, summed with its partner's copy; lane l ends with the
  // warp sums of outputs 2l and 2l + 1
#pragma unroll
  for (int s = kLeanDh / 2, o = 16; s >= 2; s >>= 1, o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const float send = up ? acc[i] : acc[i + s];
      const float keep = up ? acc[i + s] : acc[i];
      acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  *reinterpret_cast<float2*>(red + warp * kLeanDh + 2 * lane) = make_float2(acc[0], acc[1]);
  __syncthreads();
  if (tid < kLeanDh) {
    float a = 0.f;
#pragma unroll
    for (int w = 0; w < kLeanThreads / 32; ++w) a += red[w * kLeanDh + tid];
    p.out[static_cast<size_t>(b) * d + h * kLeanDh + tid] = (ok && n > 0) ? a : 0.f;
  }
}

// ---------------------------------------------------------------------------- projection merge
// bf16 W_KV, d_h = 64 DHB (DHB = 1 or 2), up to 16 MT sequences per launch. Grid (H, NDB),
// clusters of NDB CTAs along y; CTA (h, r) owns head h and the rows [r·DB, (r+1)·DB) of W_KV,
// DB = 256, 512 or 1024.
//   * Before the split kernel's results are awaited: barriers, TMEM, a zeroed ū operand, and the
//     first `ws` tiles of W_KV[block rows, head-h columns] (64 rows x 64 columns per TMA box,
//     128-byte swizzle) requested into a ring of `ws` stages.
//   * The slot range of the launch's sequences, every slot's m and l and its sequence.
//   * ū[b, block] = Σ_c w_c U_c[block]: thread t owns DB/256 columns and keeps 64 floats of
//     partial rows in flight (plain loads, no barrier: the rows were just written by the split
//     kernel and are read once, so what matters is having many requests outstanding); the merge
//     weights w_c = 2^(m_c - M) / Σ 2^(m_c' - M) l_c' are formed, one warp per sequence, while the
//     first rows are in flight. Rows are added in slot order (a fixed order: deterministic); when a
//     sequence's last row has been added its sum is written as the bf16 high and low parts of the
//     MMA operand (K-major, 128-byte swizzle), so that the projection keeps fp32 accuracy on bf16
//     tensor ops.
//   * o_r = W_KV[block, h-cols]^T · ū^T on tcgen05 (M = d_h, N = 16 MT sequences, K = 16 rows of
//     the block per MMA; W_KV read in place from the ring as the MN-major operand, the high and
//     low parts accumulated into one fp32 TMEM accumulator), a ring stage refilled three stages
//     after its MMAs were issued.
//   * The NDB products of an output element are pushed to one owner CTA through distributed
//     shared memory and added there in a fixed order, so the result does not depend on timing.
struct MergeProjParams {
  const float* U;
  const float* m;
  const float* l;
  const int32_t* meta;
  float* out;
  int32_t* lens;
  int32_t* status;
  int B, d, H, ndb, max_items;
  int b_begin, nb;  // sequences of this launch (nb <= 16 MT)
  int ws;           // W_KV ring stages
};

constexpr int kProjThreads = 256;
constexpr int kProjWarps = kProjThreads / 32;
constexpr int kProjWRows = 64;       // W_KV rows per ring stage
constexpr int kProjMaxWStages = 16;  // W_KV ring stages at most
constexpr int kProjDepth = 64;       // partial-row floats in flight per thread

struct ProjSmem {
  uint32_t w, ub, part, recv, per, wts, ls, rseq, soff, bars, slot, total;
};
// BP = 16 MT sequences (the MMA's N)
__host__ __device__ inline ProjSmem proj_smem_layout(int DB, int d_h, int nb, int ndb, int ws, int max_items) {
  ProjSmem s;
  const uint32_t BP = up_to(static_cast<uint32_t>(nb), 16u);
  uint32_t o = 0;
  s.w = o;  // [ws][d_h / 64 boxes][64 rows][128 bytes]
  o += static_cast<uint32_t>(ws) * kProjWRows * d_h * 2u;
  s.ub = o;  // ū in bf16, high then low part: [2][DB / 64 chunks][BP rows][128 bytes], swizzled
  o += 2u * static_cast<uint32_t>(DB) * BP * 2u;
  s.part = o;  // this CTA's products [nb][d_h]
  o += up_to(static_cast<uint32_t>(nb) * d_h * 4u, 16u);
  s.per = (static_cast<uint32_t>(nb) * d_h + ndb - 1u) / ndb;
  s.recv = o;  // products pushed by the cluster's CTAs: [ndb][per]
  o += up_to(static_cast<uint32_t>(ndb) * s.per * 4u, 16u);
  s.wts = o;  // m of every slot of the launch, then its merge weight
  o += up_to(static_cast<uint32_t>(max_items), 4u) * 4u;
  s.ls = o;  // l of every slot of the launch
  o += up_to(static_cast<uint32_t>(max_items), 4u) * 4u;
  s.rseq = o;  // sequence (within the launch) of every slot
  o += up_to(static_cast<uint32_t>(max_items), 4u) * 4u;
  s.soff = o;
  o += up_to(static_cast<uint32_t>(nb) + 1u, 4u) * 4u;
  o = up_to(o, 8u);
  s.bars = o;  // wfull [ws], wempty [ws], accbar
  o += (2u * static_cast<uint32_t>(ws) + 1u) * 8u;
  s.slot = o;  // TMEM address, failure flag
  o += 16u;
  s.total = o + 1024u;  // slack to align the base to 1024 bytes
  return s;
}

// Byte offset of ū[n][k] in one K-major, 128-byte-swizzled operand part [DB/64][BP][128 B].
__device__ __forceinline__ uint32_t proj_ub_off(int n, int k, int BP) {
  return static_cast<uint32_t>((k >> 6) * (BP * 128) + n * 128 + ((((k & 63) >> 3) ^ (n & 7)) << 4) + (k & 7) * 2);
}

// ū rows of the launch's sequences from their slots, VEC columns per thread: kProjDepth / VEC
// rows in flight; `prep` runs once the first rows are requested, `flush(seq, acc)` receives each
// sequence's finished sum.
template <int VEC, typename Prep, typename Flush>
__device__ __forceinline__ void proj_sum_rows(const float* ubase, size_t ustride, int nrows, const int* rseq,
                                              const float* wts, int tid, Prep prep, Flush flush) {
  constexpr int D = kProjDepth / VEC;
  typedef typename std::conditional<VEC == 4, float4, typename std::conditional<VEC == 2, float2, float>::type>::type
      VT;
  const VT* src = reinterpret_cast<const VT*>(ubase) + tid;
  const size_t vstride = ustride / VEC;
  float acc[VEC];
#pragma unroll
  for (int k = 0; k < VEC; ++k) acc[k] = 0.f;
  int cur = -1;
  if (nrows == 0) prep();
#pragma unroll 1
  for (int c0 = 0; c0 < nrows; c0 += D) {
    VT v[D];
#pragma unroll
    for (int u = 0; u < D; ++u) {
      if (c0 + u < nrows) v[u] = __ldcg(src + static_cast<size_t>(c0 + u) * vstride);
    }
    if (c0 == 0) prep();  // the merge weights, while the first rows are in flight
#pragma unroll
    for (int u = 0; u < D; ++u) {
      const int c = c0 + u;
      if (c >= nrows) break;
      const int sq = rseq[c];
      if (sq != cur) {
        if (cur >= 0) flush(cur, acc);
        cur = sq;
#pragma unroll
        for (int k = 0; k < VEC; ++k) acc[k] = 0.f;
      }
      const float w = wts[c];
      const float* x = reinterpret_cast<const float*>(&v[u]);
#pragma unroll
      for (int k = 0; k < VEC; ++k) acc[k] = fmaf(w, x[k], acc[k]);
    }
  }
  if (cur >= 0) flush(cur, acc);
}

template <int DHB, int MT>
__global__ void __launch_bounds__(kProjThreads, 1)
    merge_proj_kernel(const __grid_constant__ CUtensorMap wmap, const MergeProjParams p) {
  extern __shared__ uint8_t psm_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(psm_raw) + 1023) & ~uintptr_t(1023));
  constexpr int DH = 64 * DHB;
  constexpr int BP = 16 * MT;                         // N of the projection MMA
  constexpr uint32_t kTmemCols = BP <= 32 ? 32 : 64;  // fp32 accumulator columns
  const int h = blockIdx.x, r = blockIdx.y;
  const int DB = p.d / p.ndb, c0 = r * DB;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nb = p.nb, b0 = p.b_begin, WS = p.ws;
  const ProjSmem L = proj_smem_layout(DB, DH, nb, p.ndb, WS, p.max_items);
  uint8_t* wring = sm + L.w;
  uint8_t* ubhi = sm + L.ub;
  uint8_t* ublo = ubhi + static_cast<uint32_t>(DB) * BP * 2u;
  float* part = reinterpret_cast<float*>(sm + L.part);
  float* recv = reinterpret_cast<float*>(sm + L.recv);
  float* wts = reinterpret_cast<float*>(sm + L.wts);
  float* ls = reinterpret_cast<float*>(sm + L.ls);
  int* rseq = reinterpret_cast<int*>(sm + L.rseq);
  int* s_off = reinterpret_cast<int*>(sm + L.soff);
  uint64_t* wfull = reinterpret_cast<uint64_t*>(sm + L.bars);
  uint64_t* wempty = wfull + WS;  // the MMAs of the stage completed
  uint64_t* accbar = wempty + WS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L.slot);
  int* fail = reinterpret_cast<int*>(sm + L.slot + 4);
  const int nws = DB / kProjWRows;  // W_KV stages of this block
  constexpr uint32_t kWStageBytes = kProjWRows * DH * 2u;

  int w_issued = 0;  // thread 0 issues every W_KV copy and MMA
  auto issue_w = [&](int st) {  // W_KV rows c0 + 64 st .., head-h columns, into ring stage st % WS
    uint8_t* dst = wring + (st % WS) * kWStageBytes;
    uint64_t* bar = &wfull[st % WS];
    mbar_arrive_expect_tx(bar, kWStageBytes);
#pragma unroll
    for (int wb = 0; wb < DHB; ++wb)
      tma_load_2d(dst + wb * kProjWRows * 128, &wmap, h * DH + wb * 64, c0 + st * kProjWRows, bar,
                  l2_policy_evict_first());
    ++w_issued;
  };

  // ---- before the split kernel's results exist
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  } else if (warp == 1 && lane == 0) {
    for (int s = 0; s < WS; ++s) {
      mbar_init(&wfull[s], 1);
      mbar_init(&wempty[s], 1);
    }
    mbar_init(accbar, 1);
    *fail = 0;
    fence_barrier_init();
  }
  {
    uint4* z = reinterpret_cast<uint4*>(ubhi);  // operand rows of absent sequences stay zero
    const int n16 = static_cast<int>(2u * static_cast<uint32_t>(DB) * BP * 2u / 16u);
    for (int i = tid; i < n16; i += kProjThreads) z[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (tid == 0) {
    tma_prefetch_desc(&wmap);
    for (int st = 0; st < min(WS, nws); ++st) issue_w(st);
  }
  if (p.ndb > 1) cluster_arrive_relaxed();
  pdl_wait_primary();
  pdl_launch_dependents();

  // ---- slot ranges of the launch's sequences; the lengths advance once (CTA (0, 0))
  for (int i = tid; i <= nb; i += kProjThreads) s_off[i] = __ldcg(p.meta + 1 + b0 + i);
  if (h == 0 && r == 0)
    for (int b = b0 + tid; b < b0 + nb; b += kProjThreads)
      if (__ldcg(p.meta + 2 + p.B + b) & kSeqAppend) p.lens[b] += 1;
  __syncthreads();
  const int s_beg = s_off[0], nrows = s_off[nb] - s_beg;

  // ---- m and l of every slot (one load each, all in flight together) and each slot's sequence
  for (int c = tid; c < nrows; c += kProjThreads) {
    wts[c] = __ldcg(p.m + static_cast<size_t>(s_beg + c) * p.H + h);
    ls[c] = __ldcg(p.l + static_cast<size_t>(s_beg + c) * p.H + h);
  }
  for (int bl = warp; bl < nb; bl += kProjWarps)
    for (int c = s_off[bl] - s_beg + lane; c < s_off[bl + 1] - s_beg; c += 32) rseq[c] = bl;
  // merge weights, one warp per sequence, from shared memory; run once the first rows are in flight
  auto weights = [&]() {
    __syncthreads();
    for (int bl = warp; bl < nb; bl += kProjWarps) {
      const int lo = s_off[bl] - s_beg, hi = s_off[bl + 1] - s_beg;
      float M = -INFINITY;
      for (int c = lo + lane; c < hi; c += 32) M = fmaxf(M, wts[c]);
      M = warp_max(M);
      float S = 0.f;
      for (int c = lo + lane; c < hi; c += 32) {
        const float e = exp2f(wts[c] - M);
        S = fmaf(e, ls[c], S);
        ls[c] = e;
      }
      S = warp_sum(S);
      const float inv = S > 0.f ? 1.f / S : 0.f;
      __syncwarp();
      for (int c = lo + lane; c < hi; c += 32) wts[c] = ls[c] * inv;
    }
    __syncthreads();
  };

  // ---- ū[b, block] = Σ_c w_c U_c[block]; each finished sequence becomes the bf16 high and low
  // operand rows
  {
    const float* ubase = p.U + (static_cast<size_t>(s_beg) * p.H + h) * p.d + c0;
    const size_t ustride = static_cast<size_t>(p.H) * p.d;  // floats between slots
    auto flush = [&](int seq, const float* acc, int vec) {
      for (int k = 0; k < vec; ++k) {
        const int col = vec * tid + k;
        const __nv_bfloat16 hi = __float2bfloat16_rn(acc[k]);
        const __nv_bfloat16 lo = __float2bfloat16_rn(acc[k] - __bfloat162float(hi));
        const uint32_t off = proj_ub_off(seq, col, BP);
        *reinterpret_cast<__nv_bfloat16*>(ubhi + off) = hi;
        *reinterpret_cast<__nv_bfloat16*>(ublo + off) = lo;
      }
    };
    if (DB == 1024)
      proj_sum_rows<4>(ubase, ustride, nrows, rseq, wts, tid, weights,
                       [&](int sq, const float (&a)[4]) { flush(sq, a, 4); });
    else if (DB == 512)
      proj_sum_rows<2>(ubase, ustride, nrows, rseq, wts, tid, weights,
                       [&](int sq, const float (&a)[2]) { flush(sq, a, 2); });
    else
      proj_sum_rows<1>(ubase, ustride, nrows, rseq, wts, tid, weights,
                       [&](int sq, const float (&a)[1]) { flush(sq, a, 1); });
  }
  fence_proxy_async_smem();  // the operand is read by the tensor cores (async proxy)
  __syncthreads();

  // ---- o_r = W_KV[block, h-cols]^T · ū^T on tcgen05
  if (tid == 0) {
    const uint32_t idesc = idesc_bf16_f32(static_cast<uint32_t>(DH), static_cast<uint32_t>(BP), 1u, 0u);
    const uint32_t wbase = smem_u32(wring), hib = smem_u32(ubhi), lob = smem_u32(ublo);
    const int lag = min(3, WS - 1);
    bool ok = true;
    int done = 0;  // stages whose copies were waited for
    for (int st = 0; st < nws; ++st) {
      if (!mbar_wait(&wfull[st % WS], static_cast<uint32_t>(st / WS) & 1u, p.status)) {
        ok = false;
        break;
      }
      done = st + 1;
      tc_fence_after();
      const uint32_t ws_ = wbase + (st % WS) * kWStageBytes;
#pragma unroll
      for (int kk = 0; kk < kProjWRows / 16; ++kk) {
        // A: MN-major (d_h contiguous), 64-column blocks 64 rows x 128 B (8 KB) apart, 8-row groups
        // 1024 B apart, a 16-row step is 2 KB. B: K-major rows of 128 B, 8-row groups 1024 B apart,
        // a 16-column step is 32 B, a 64-column chunk is BP x 128 B.
        const uint64_t ad = smem_desc(ws_ + kk * 2048, kProjWRows * 128, 1024, kLayoutSW128);
        const uint32_t boff = st * (BP * 128) + kk * 32;
        umma_f16(tmem, ad, smem_desc(hib + boff, 16, 1024, kLayoutSW128), idesc, (st > 0 || kk > 0) ? 1u : 0u);
        umma_f16(tmem, ad, smem_desc(lob + boff, 16, 1024, kLayoutSW128), idesc, 1u);
      }
      umma_commit(&wempty[st % WS]);
      // refill the stage used `lag` stages ago: its MMAs have completed by now, so the refill does
      // not wait on the tensor pipe (stage st - lag + WS is needed only lag - WS stages later)
      const int jw = st - lag;
      if (jw >= 0 && jw + WS < nws) {
        if (!mbar_wait(&wempty[jw % WS], static_cast<uint32_t>(jw / WS) & 1u, p.status)) {
          ok = false;
          break;
        }
        issue_w(jw + WS);
      }
    }
    umma_commit(accbar);  // also after a failure: covers every MMA issued
    if (!ok) {
      *fail = 1;
      // copies still landing in this CTA's shared memory must complete before it exits
      for (int st = done; st < w_issued; ++st)
        mbar_wait(&wfull[st % WS], static_cast<uint32_t>(st / WS) & 1u, p.status);
    }
  }
  __syncwarp();
  bool ok = mbar_wait(accbar, 0u, p.status);
  ok = __syncthreads_and(ok) && *fail == 0;
  tc_fence_after();
  // accumulator row n (output column n of the head) holds the BP sequences' values
  if (warp < 4) {
    const bool has_row = DH == 128 || lane < 16;  // M = 64: lanes 16..31 of a quarter are unused
    const int n = DH == 128 ? warp * 32 + lane : warp * 16 + lane;
#pragma unroll
    for (int cb = 0; cb < BP; cb += 16) {
      float v[16];
      tmem_ld16(tmem + (static_cast<uint32_t>(warp * 32) << 16) + static_cast<uint32_t>(cb), v);
      tmem_wait_ld();
      if (has_row) {
#pragma unroll
        for (int e = 0; e < 16; ++e)
          if (cb + e < nb) part[(cb + e) * DH + n] = ok ? v[e] : 0.f;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }

  // ---- sum the NDB products: push each element to its owner CTA, then add in a fixed order
  const int n_out = nb * DH;
  if (p.ndb == 1) {
    for (int e = tid; e < n_out; e += kProjThreads)
      p.out[static_cast<size_t>(b0 + e / DH) * p.d + h * DH + e % DH] = part[e];
    return;
  }
  cluster_wait();  // every CTA of the cluster is running
  const uint32_t recv_base = smem_u32(recv);
  const int per = static_cast<int>(L.per);
  for (int e = tid; e < n_out; e += kProjThreads)
    st_cluster_f32(mapa_shared(recv_base + 4u * static_cast<uint32_t>(r * per + e / p.ndb), e % p.ndb), part[e]);
  cluster_sync();  // pushes visible; nobody touches a peer's shared memory after this
  for (int s2 = tid; s2 < per; s2 += kProjThreads) {
    const int e = s2 * p.ndb + r;
    if (e >= n_out) break;
    float a = 0.f;
    for (int q = 0; q < p.ndb; ++q) a += recv[q * per + s2];
    p.out[static_cast<size_t>(b0 + e / DH) * p.d + h * DH + e % DH] = a;
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

struct MergeConfig {
  int ndb, nb_max;
  size_t smem;
};

// CUDA-core merge: NDB the smallest of 1, 2, 4, 8 that gives at least one CTA per SM,
// preferring a footprint that lets two CTAs share an SM; 16 (a non-portable cluster) only
// when no smaller block fits.
bool pick_merge(int B, int d, int H, int esz, int max_items, MergeConfig* c) {
  const int d_h = d / H;
  if (d_h % 4 || (d_h * esz) % 16 || d_h > 256) return false;
  c->nb_max = kMergeMaxSeqs;
  const int nb = std::min(B, c->nb_max);
  const size_t half = static_cast<size_t>(max_smem_optin()) / 2 - 2048, full = static_cast<size_t>(max_smem_optin()) - 2048;
  // rank 3: enough CTAs and two per SM; 2: enough CTAs; 1: fits (the most blocks wins)
  int best = 0, best_rank = 0;
  size_t best_smem = 0;
  for (int ndb = 1; ndb <= 16; ndb *= 2) {
    if (ndb == 16 && best != 0) break;
    if (d % ndb) break;
    const int DB = d / ndb;
    if (DB % 4 || (DB > 256 && DB % 256) || DB / 4 > kMergeThreads) continue;
    const size_t sm = merge_smem_layout(DB, d_h, esz, nb, ndb, max_items).total;
    if (sm > full) continue;
    const bool enough = H * ndb >= num_sms();
    const int rank = enough ? (sm <= half ? 3 : 2) : 1;
    if (rank > best_rank || (rank == 1 && best_rank == 1)) {
      best = ndb;
      best_rank = rank;
      best_smem = sm;
    }
    if (rank == 3) break;
  }
  if (best == 0) return false;
  c->ndb = best;
  c->smem = best_smem;
  return true;
}

struct ProjConfig {
  int ndb, ws, nb_max;
  uint32_t smem;
};

template <int DHB, int MT>
int proj_resident_clusters(int ndb, uint32_t smem, int H) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(H), static_cast<unsigned>(ndb), 1);
  cfg.blockDim = dim3(kProjThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = static_cast<unsigned>(ndb);
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  auto kern = merge_proj_kernel<DHB, MT>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

int proj_resident(int dhb, int mt, int ndb, uint32_t smem, int H) {
#define SLIM_PROJ_RES(D_, M_) \
  if (dhb == D_ && mt == M_) return proj_resident_clusters<D_, M_>(ndb, smem, H);
  SLIM_PROJ_RES(1, 1) SLIM_PROJ_RES(1, 2) SLIM_PROJ_RES(1, 3) SLIM_PROJ_RES(1, 4)
  SLIM_PROJ_RES(2, 1) SLIM_PROJ_RES(2, 2) SLIM_PROJ_RES(2, 3) SLIM_PROJ_RES(2, 4)
#undef SLIM_PROJ_RES
  return 0;
}

// Projection merge for bf16 W_KV and d_h = 64 or 128. Up to 64 sequences per launch (fewer when
// the operand does not fit). NDB (1..8, DB = d/NDB of 256, 512 or 1024 columns) and the W_KV ring
// depth are chosen so that the H x NDB CTAs run in one wave with as many CTAs as possible (a
// shallower ring that lets two CTAs share an SM counts), then the deepest ring, then the fewest
// blocks.
bool pick_proj_uncached(int B, int d, int H, int max_items, ProjConfig* c) {
  const int d_h = d / H;
  if (d_h != 64 && d_h != 128) return false;
  const uint32_t optin = static_cast<uint32_t>(max_smem_optin());
  for (int nb_max : {64, 32, 16}) {
    const int nb = std::min(B, nb_max);
    const int mt = (nb + 15) / 16;
    int best = 0, best_ctas = -1, best_ws = 0;
    uint32_t best_smem = 0;
    for (int ndb = 1; ndb <= 8; ++ndb) {
      if (d % ndb) continue;
      const int DB = d / ndb;
      if (DB != 256 && DB != 512 && DB != 1024) continue;
      int last_fit = -1;
      for (int ws = std::min(kProjMaxWStages, DB / kProjWRows); ws >= 2; --ws) {
        const uint32_t sm = proj_smem_layout(DB, d_h, nb, ndb, ws, max_items).total;
        if (sm > optin) continue;
        const int fit = proj_resident(d_h / 64, mt, ndb, sm, H);  // clusters resident at once
        if (fit <= 0 || fit == last_fit) continue;  // a shallower ring only helps if more CTAs fit
        last_fit = fit;
        const int score = H <= fit ? H * ndb : 0;  // CTAs, when all of them run in one wave
        if (score > best_ctas) {
          best = ndb;
          best_ctas = score;
          best_ws = ws;
          best_smem = sm;
        }
      }
    }
    if (best == 0) {
      if (nb < nb_max) return false;  // a smaller launch would not help
      continue;
    }
    c->ndb = best;
    c->ws = best_ws;
    c->nb_max = nb_max;
    c->smem = best_smem;
    return true;
  }
  return false;
}

// pick_proj_uncached memoised per (device, shape): it queries the occupancy API.
bool pick_proj(int B, int d, int H, int max_items, ProjConfig* c) {
  static std::mutex mu;
  static std::map<std::tuple<int, int, int, int, int>, std::pair<bool, ProjConfig>> memo;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  const auto key = std::make_tuple(dev, B, d, H, max_items);
  std::lock_guard<std::mutex> lock(mu);
  auto it = memo.find(key);
  if (it == memo.end()) {
    ProjConfig pc{};
    const bool ok = pick_proj_uncached(B, d, H, max_items, &pc);
    it = memo.emplace(key, std::make_pair(ok, pc)).first;
  }
  *c = it->second.second;
  return it->second.first;
}

}  // namespace

namespace {

// Rows of U staged per round by merge_lean_kernel for this shape, 0 if it does not apply.
int lean_cap_items(int B, int d, int H, int dtype, int max_items) {
  if (dtype != SLIM_BF16 || H * kLeanDh != d || d % kLeanThreads || d > kLeanMaxCols) return 0;
  if (static_cast<long long>(B) * H > num_sms()) return 0;  // one wave (one CTA per SM)
  if (max_items > 32 * kLeanWBlk) return 0;                  // items' merge weights: one per thread
  const int optin = max_smem_optin();
  const uint32_t fixed = lean_smem_layout(d, 0, max_items).total;
  if (fixed >= static_cast<uint32_t>(optin)) return 0;
  const int cap = std::min(32, static_cast<int>((static_cast<uint32_t>(optin) - fixed) / (static_cast<uint32_t>(d) * 4u)));
  return cap >= 4 ? cap : 0;
}

cudaError_t launch_merge_lean(const DecodeArgs& a, const SplitWorkspace& ws, int cap, bool pdl, cudaStream_t st,
                              int* launches) {
  CUtensorMap wmap;
  const uint64_t dims[2] = {static_cast<uint64_t>(a.d), static_cast<uint64_t>(a.d)};
  const uint64_t strides[1] = {static_cast<uint64_t>(a.d) * 2u};
  const uint32_t box[2] = {static_cast<uint32_t>(kLeanDh), 256u};
  if (!encode_tmap(&wmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.w_kv, dims, strides, box, true))
    return cudaErrorInvalidValue;
  MergeLeanParams p;
  p.U = ws.U;
  p.m = ws.m;
  p.l = ws.l;
  p.meta = ws.meta;
  p.out = a.out;
  p.lens = a.lens;
  p.status = a.status;
  p.B = a.B;
  p.d = a.d;
  p.H = a.H;
  p.max_items = ws.max_items;
  p.cap_items = cap;
  const uint32_t smem = lean_smem_layout(a.d, cap, ws.max_items).total;
  cudaError_t e = cudaFuncSetAttribute(merge_lean_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.H), static_cast<unsigned>(a.B), 1);
  cfg.blockDim = dim3(kLeanThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, merge_lean_kernel, wmap, p);
  if (e == cudaSuccess && launches) ++*launches;
  return e;
}

}  // namespace

namespace {

template <int DHB, int MT>
cudaError_t launch_proj_instance(const CUtensorMap& wmap, const MergeProjParams& p, uint32_t smem, bool pdl,
                                 cudaStream_t st) {
  auto kern = merge_proj_kernel<DHB, MT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.H), static_cast<unsigned>(p.ndb), 1);
  cfg.blockDim = dim3(kProjThreads, 1, 1);
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
  return cudaLaunchKernelEx(&cfg, kern, wmap, p);
}

cudaError_t launch_merge_proj(const DecodeArgs& a, const SplitWorkspace& ws, const ProjConfig& c, bool pdl,
                              cudaStream_t st, int* launches) {
  const int d_h = a.d / a.H, DB = a.d / c.ndb;
  // W_KV as {d columns, d rows}, bf16; a box is 64 columns x 64 rows, 128-byte swizzled
  CUtensorMap wmap;
  const uint64_t dims[2] = {static_cast<uint64_t>(a.d), static_cast<uint64_t>(a.d)};
  const uint64_t strides[1] = {static_cast<uint64_t>(a.d) * 2u};
  const uint32_t box[2] = {64u, static_cast<uint32_t>(kProjWRows)};
  if (!encode_tmap(&wmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.w_kv, dims, strides, box, true))
    return cudaErrorInvalidValue;
  for (int b0 = 0; b0 < a.B; b0 += c.nb_max) {
    MergeProjParams p;
    p.U = ws.U;
    p.m = ws.m;
    p.l = ws.l;
    p.meta = ws.meta;
    p.out = a.out;
    p.lens = a.lens;
    p.status = a.status;
    p.B = a.B;
    p.d = a.d;
    p.H = a.H;
    p.ndb = c.ndb;
    p.max_items = ws.max_items;
    p.b_begin = b0;
    p.nb = std::min(c.nb_max, a.B - b0);
    p.ws = c.ws;
    const int mt = (p.nb + 15) / 16;
    const uint32_t smem = proj_smem_layout(DB, d_h, p.nb, c.ndb, c.ws, ws.max_items).total;
    const bool dep = pdl && b0 == 0;
    cudaError_t e = cudaErrorNotSupported;
#define SLIM_PROJ_CASE(D_, M_) \
    if (d_h == 64 * D_ && mt == M_) e = launch_proj_instance<D_, M_>(wmap, p, smem, dep, st);
    SLIM_PROJ_CASE(1, 1) SLIM_PROJ_CASE(1, 2) SLIM_PROJ_CASE(1, 3) SLIM_PROJ_CASE(1, 4)
    SLIM_PROJ_CASE(2, 1) SLIM_PROJ_CASE(2, 2) SLIM_PROJ_CASE(2, 3) SLIM_PROJ_CASE(2, 4)
#undef SLIM_PROJ_CASE
    if (e != cudaSuccess) return e;
    if (launches) ++*launches;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_reduce_b(const DecodeArgs& a, const SplitWorkspace& ws, bool pdl, cudaStream_t st,
                            int* launches) {
  if (const int cap = lean_cap_items(a.B, a.d, a.H, a.dtype, ws.max_items))
    return launch_merge_lean(a, ws, cap, pdl, st, launches);
  if (a.dtype == SLIM_BF16) {
    ProjConfig pc;
    if (pick_proj(a.B, a.d, a.H, ws.max_items, &pc)) return launch_merge_proj(a, ws, pc, pdl, st, launches);
  }
  const int esz = a.dtype == SLIM_BF16 ? 2 : 4;
  const int d_h = a.d / a.H;
  MergeConfig c;
  if (!pick_merge(a.B, a.d, a.H, esz, ws.max_items, &c)) return cudaErrorNotSupported;
  const int DB = a.d / c.ndb;
  // W_KV as {d columns, d rows}; a box is the head's d_h columns x up to 256 rows, dense
  CUtensorMap wmap;
  const uint64_t dims[2] = {static_cast<uint64_t>(a.d), static_cast<uint64_t>(a.d)};
  const uint64_t strides[1] = {static_cast<uint64_t>(a.d) * esz};
  const uint32_t box[2] = {static_cast<uint32_t>(d_h), static_cast<uint32_t>(std::min(DB, 256))};
  if (!encode_tmap(&wmap, esz == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, a.w_kv,
                   dims, strides, box, false))
    return cudaErrorInvalidValue;
  auto kern = (a.dtype == SLIM_BF16) ? merge_b_kernel<__nv_bfloat16> : merge_b_kernel<float>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(c.smem));
  if (e == cudaSuccess && c.ndb > 8) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e != cudaSuccess) return e;
  for (int b0 = 0; b0 < a.B; b0 += c.nb_max) {
    MergeBParams p;
    p.U = ws.U;
    p.m = ws.m;
    p.l = ws.l;
    p.meta = ws.meta;
    p.out = a.out;
    p.lens = a.lens;
    p.status = a.status;
    p.B = a.B;
    p.d = a.d;
    p.H = a.H;
    p.ndb = c.ndb;
    p.max_items = ws.max_items;
    p.b_begin = b0;
    p.nb = std::min(c.nb_max, a.B - b0);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(a.H), static_cast<unsigned>(c.ndb), 1);
    cfg.blockDim = dim3(kMergeThreads, 1, 1);
    cfg.dynamicSmemBytes = merge_smem_layout(DB, d_h, esz, p.nb, c.ndb, ws.max_items).total;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = static_cast<unsigned>(c.ndb);
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = (pdl && b0 == 0) ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, kern, wmap, p);
    if (e != cudaSuccess) return e;
    if (launches) ++*launches;
  }
  return cudaSuccess;
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
