// Generation step, ordering (b), on tensor cores (bf16 K cache).
//
// Slim Attention article, section "K-Cache is All You Need", generation
// phase, second option: multiply the per-head softmax rows by K first (a full
// d-row per head) and only then by W_KV. Per segment (the rows of one
// sequence within a work group's contiguous share of all attended rows, see
// split_plan.cuh) this kernel streams the segment's K rows once and produces
// the flash-decoding partial of every head h:
//     m_h = running max of the scaled scores (log2 domain)
//     l_h = sum_t 2^(s_ht - m_h)
//     U_h = sum_t 2^(s_ht - m_h) · K_t            (a full d-row, fp32)
// reduce.cu merges the partials and applies W_KV.
//
// A cluster of CL CTAs is one work group; CTA r owns the columns
// [r·dS, (r+1)·dS), dS = d/CL <= 1024, and the heads whose columns lie there.
// Per CTA (16 warps):
//   warp 0       TMA producer: a K tile is TT rows x dS columns, one 3-D box
//                per 16-row slab (128-byte swizzle), evict-first in L2.
//   warp 1       MMA issuer: U[heads, own columns] += P[heads, rows] · K[rows,
//                own columns] with tcgen05.mma kind::f16, M = 64 (heads),
//                N <= 256 (columns), K = 16 rows; the K slab is read in place
//                as the MN-major B operand. Two M=64 accumulators interleave in
//                TMEM (lane offsets 0 and 16), so 1024 columns fit in the 512
//                TMEM columns.
//   warps 2..5   correction and epilogue: the lazy online-softmax rescale of
//                the accumulator rows whose max grew by more than 2^8 (the MMA
//                warp waits for this pass first only on tiles with a rescaled
//                row), and TMEM -> partials in global memory.
//   warps 6..15  scores: per head, q_h·K_t on the CUDA cores (32-row tiles: a
//                lane multiplies one 16-byte chunk of 8 rows by q held in
//                registers, a butterfly over the 8 chunk lanes sums the rows;
//                16-row tiles: one row per lane, q broadcast from shared
//                memory), fp32 accumulation, running max, P in bf16 and the
//                rescale factors to this CTA's rows of the stage. With CL > 1
//                the same warps store those rows into every peer with st.async
//                (16 bytes of P per store), which completes the bytes on the
//                peer's mbarrier: no fence and no round trip on the sending
//                side, and the stores do not queue behind the TMA unit's K
//                loads as a bulk copy would. The tensor pipe is left to the
//                P·K MMAs. Ten warps, so that 10 heads (d=1280, H=20 split
//                over two CTAs) take one warp each.
// Every mbarrier wait is bounded; a timeout sets SLIM_DEV_TIMEOUT and the
// kernel drains its copies and MMAs, frees TMEM and returns.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstdlib>
#include <map>
#include <mutex>
#include <utility>

#include "split_plan.cuh"

namespace slim {

// A head's running max may grow by this much (log2 units) before its TMEM row
// is rescaled: P stays <= 2^8 in bf16 and no precision is lost.
constexpr float kLazyRescaleLog2 = 8.f;
constexpr int kSoftmaxWarps = 10;
constexpr int kTCThreads = (6 + kSoftmaxWarps) * 32;
constexpr int kMaxColsPerCTA = 1024;  // two interleaved M=64 accumulators x 512 TMEM columns
constexpr int kPRows = 64;            // M of the P·K MMA: heads, padded

struct DecodeTCParams {
  const float* q;
  const __nv_bfloat16* k_new;
  __nv_bfloat16* kcache;
  const int32_t* lens;
  int32_t* status;
  float* ws_U;
  float* ws_m;
  float* ws_l;
  int32_t* ws_meta;
  int B, d, H;
  int64_t cap;
  int append;
  int n_groups;   // clusters launched
  int stages;
  int min_rows;
  uint32_t tmem_cols;
  float scale_log2;
  uint64_t wait_ns;  // limit of every wait (kWaitLimitNs unless a test shortens it)
  int stall;         // test hook: the MMA warp first waits on a barrier nothing completes
};

// Shared-memory carve-up, identical on host and device.
struct TCSmem {
  uint32_t k_off, p_off, alpha_off, q_off, bar_off, slot_off, plan_off, total;
};
__host__ __device__ inline TCSmem tc_smem_layout(int CL, int TT, int d, int stages, int B) {
  TCSmem s;
  const uint32_t dS = static_cast<uint32_t>(d / CL);
  uint32_t o = 0;
  s.k_off = o;
  o += static_cast<uint32_t>(stages) * TT * dS * 2u;
  s.p_off = o;
  o += static_cast<uint32_t>(stages) * kPRows * TT * 2u;
  s.alpha_off = o;  // per stage: the rescale factor of every P row (1 = none)
  o += static_cast<uint32_t>(stages) * kPRows * 4u;
  s.q_off = o;
  o += dS * 4u;
  o = (o + 7u) & ~7u;
  s.bar_off = o;
  o += (5u * stages + 3u) * 8u;
  s.slot_off = o;
  o += 16u;
  s.plan_off = o;  // s_nb [B + 1], s_q [B + 1], s_soff [B + 1], s_plan [2]
  o += (3u * static_cast<uint32_t>(B + 1) + 2u) * 4u;
  s.total = o + 1024u;  // slack for aligning the base to 1024 bytes
  return s;
}

// Row of head n in the P operand and the accumulator. CTA r of a cluster owns
// heads [r·H_own, (r+1)·H_own) and the contiguous rows [r·64/CL, (r+1)·64/CL),
// so its part of P (and of alpha) is one block it can copy to its peers. The
// 16-row TMEM lane quarters of that block take its heads in turn (j, j + 4/CL,
// ... share a quarter), so the four correction warps split the rows evenly.
__host__ __device__ inline int p_row(int n, int CL, int H_own) {
  const int qpr = 4 / CL, r = n / H_own, j = n - r * H_own;
  return r * (kPRows / CL) + 16 * (j % qpr) + j / qpr;
}
// The inverse: the head in row i, or -1 for a padding row.
__host__ __device__ inline int row_head(int i, int CL, int H_own) {
  const int R = kPRows / CL, qpr = 4 / CL, r = i / R, w = i - r * R;
  const int j = (w % 16) * qpr + w / 16;
  return j < H_own ? r * H_own + j : -1;
}

// Softmax warps are warps 6 .. 6 + kSoftmaxWarps - 1; warp w issues on sub-partition w % 4.
// The SMSP-balanced assignment gives head j to sub-partition j % 4 and, within it, to its
// softmax warps in turn, so every sub-partition issues about H_own / 4 heads' score work (the
// plain assignment, heads sw, sw + kSoftmaxWarps, ..., leaves 5 of 16 heads on two of them).
// It is used when no warp then needs more than HPW heads.
__host__ __device__ inline void smsp_warps(int x, int* first, int* len) {
  *first = 6 + ((x + 2) & 3);
  *len = (6 + kSoftmaxWarps - *first + 3) / 4;
}
__host__ __device__ inline bool balanced_heads_fit(int H_own, int HPW) {
  for (int x = 0; x < 4; ++x) {
    int first, len;
    smsp_warps(x, &first, &len);
    const int n = H_own > x ? (H_own - x + 3) / 4 : 0;
    if ((n + len - 1) / len > HPW) return false;
  }
  return true;
}
// Head of softmax warp sw in slot k, or H_own when the slot is empty.
__host__ __device__ inline int softmax_head(int sw, int k, int H_own, bool balanced) {
  int j;
  if (balanced) {
    const int w = sw + 6, x = w & 3;
    int first, len;
    smsp_warps(x, &first, &len);
    j = x + 4 * ((w - first) / 4 + len * k);
  } else {
    j = sw + kSoftmaxWarps * k;
  }
  return j < H_own ? j : H_own;
}

template <int CL, int TT, int DHB, int HPW>
__global__ void __launch_bounds__(kTCThreads, 1)
    decode_b_tc_kernel(const __grid_constant__ CUtensorMap kmap, const DecodeTCParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int DH = DHB * 64;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = (CL > 1) ? cluster_ctarank() : 0u;
  const int group = blockIdx.x / CL;
  const int dS = p.d / CL, col0 = static_cast<int>(rank) * dS;
  const int ncb = dS / 64;
  const int H_own = p.H / CL, head0 = static_cast<int>(rank) * H_own;
  const int stages = p.stages;
  const TCSmem L = tc_smem_layout(CL, TT, p.d, stages, p.B);
  uint8_t* kst = smem + L.k_off;
  uint8_t* pst = smem + L.p_off;
  float* alpha_s = reinterpret_cast<float*>(smem + L.alpha_off);  // [stages][kPRows], by P row
  float* q_s = reinterpret_cast<float*>(smem + L.q_off);  // this CTA's columns of q
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* full = bars;                       // TMA landed (tx bytes)
  uint64_t* empty = bars + stages;             // this CTA's MMAs done with the K stage
  uint64_t* pfull = bars + 2 * stages;         // P and alpha of every head of the cluster in place
  uint64_t* pempty = bars + 3 * stages;        // every CTA's MMAs done with the P stage, alphas read
  uint64_t* corr = bars + 4 * stages;          // accumulator corrected for this tile's new maxima
  uint64_t* accfull = bars + 5 * stages;       // last MMA of a segment completed
  uint64_t* accempty = bars + 5 * stages + 1;  // epilogue finished reading the accumulator
  uint64_t* stallbar = bars + 5 * stages + 2;  // test hook: never completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.slot_off);
  int* s_nb = reinterpret_cast<int*>(smem + L.plan_off);
  unsigned* s_q = reinterpret_cast<unsigned*>(s_nb + (p.B + 1));
  unsigned* s_soff = s_q + (p.B + 1);
  unsigned* s_plan = s_soff + (p.B + 1);
  const uint32_t kstage_bytes = static_cast<uint32_t>(TT) * dS * 2u;
  const uint32_t pstage_bytes = static_cast<uint32_t>(kPRows) * TT * 2u;
  // K stage layout: [TT/16 slabs][ncb column blocks][16 rows][128 bytes], 128-byte swizzled
  const uint32_t slab_bytes = static_cast<uint32_t>(ncb) * 2048u;

  // ---------------------------------------------------------------- set-up
  // Nothing before pdl_wait_primary() reads memory that earlier work in the
  // stream may still be writing (lengths, caches, queries, workspace).
  if (warp == 0) {
    if (lane == 0) tma_prefetch_desc(&kmap);
  } else if (warp == 1) {
    if (lane == 0) {
      for (int s = 0; s < stages; ++s) {
        mbar_init(&full[s], 1);
        mbar_init(&empty[s], 1);
        // one arrival per softmax warp; with peers, one of them also expects the peers'
        // P rows and alphas as transaction bytes
        mbar_init(&pfull[s], kSoftmaxWarps);
        mbar_init(&pempty[s], CL);
        mbar_init(&corr[s], 4);
      }
      mbar_init(accfull, 1);
      mbar_init(accempty, 4);
      mbar_init(stallbar, 1);
      fence_barrier_init();
    }
    __syncwarp();
    tmem_alloc(tmem_slot, p.tmem_cols);
    tmem_relinquish();
  } else if (warp >= 6) {
    // P buffers start at zero (rows of absent heads stay zero); every alpha starts at 1.
    const int t = threadIdx.x - 6 * 32;
    uint32_t* pz = reinterpret_cast<uint32_t*>(pst);
    for (uint32_t i = t; i < stages * pstage_bytes / 4u; i += kSoftmaxWarps * 32) pz[i] = 0u;
    for (int i = t; i < stages * kPRows; i += kSoftmaxWarps * 32) alpha_s[i] = 1.0f;
    fence_proxy_async_smem();
  }
  pdl_wait_primary();
  pdl_launch_dependents();
  if (warp == 0)
    plan_lean(p.lens, p.B, 1, p.cap, p.append, p.n_groups, p.min_rows, s_nb, s_q, s_soff, s_plan, p.ws_meta, p.status,
              blockIdx.x == 0);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (CL > 1) cluster_sync();
  const uint32_t tmem = *tmem_slot;
  LeanCursor cur;  // this group's segments (every role walks the same list)
  cur.init(group, p.B, s_q, s_plan);
  SplitItem it;
  auto tiles_of = [&](const SplitItem& it) { return (it.row1 - it.row0 + TT - 1) / TT; };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      int g = 0;  // tiles issued so far (all segments)
      bool ok = true;
      while (ok && cur.next(it, s_nb, s_q, s_soff)) {
        const int nt = tiles_of(it);
        for (int t = 0; t < nt; ++t, ++g) {
          const int s = g % stages;
          const uint32_t ph = static_cast<uint32_t>(g / stages) & 1u;
          if (g >= stages && !mbar_wait(&empty[s], ph ^ 1u, p.status, p.wait_ns)) {
            ok = false;
            break;
          }
          const int r_lo = it.row0 + t * TT;
          const int nbox = (min(TT, it.row1 - r_lo) + 15) / 16;
          mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(nbox) * slab_bytes);
          const int y0 = static_cast<int>(static_cast<int64_t>(it.b) * p.cap + r_lo);
          uint8_t* dst = kst + s * kstage_bytes;
          // one 3-D box per 16-row slab: 64 columns x 16 rows x every column block of this CTA
          for (int rb = 0; rb < nbox; ++rb)
            tma_load_3d(dst + rb * slab_bytes, &kmap, 0, y0 + rb * 16, col0 / 64, &full[s], pol);
        }
      }
      // drain: every issued copy must land before the CTA can exit
      for (int t = max(0, g - stages); t < g; ++t)
        mbar_wait(&full[t % stages], static_cast<uint32_t>(t / stages) & 1u, p.status, p.wait_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t kbase = smem_u32(kst), pbase = smem_u32(pst);
      int g = 0, ii = 0;
      // test hook: a wait that runs out before any MMA is issued; every other role then runs out
      // of its own waits, the producer drains its copies, and the kernel returns SLIM_DEV_TIMEOUT
      bool ok = !p.stall || mbar_wait(stallbar, 0u, p.status, p.wait_ns);
      while (ok && cur.next(it, s_nb, s_q, s_soff)) {
        const int nt = tiles_of(it);
        // the previous segment's epilogue must have read the accumulator
        if (ii > 0 && !mbar_wait(accempty, static_cast<uint32_t>(ii - 1) & 1u, p.status, p.wait_ns)) break;
        for (int t = 0; t < nt; ++t, ++g) {
          const int s = g % stages;
          const uint32_t ph = static_cast<uint32_t>(g / stages) & 1u;
          const uint32_t ka = kbase + s * kstage_bytes, pa = pbase + s * pstage_bytes;
          // P of every head in place and the K stage landed
          if (!mbar_wait<(CL > 1)>(&pfull[s], ph, p.status) || !mbar_wait(&full[s], ph, p.status, p.wait_ns)) {
            ok = false;
            break;
          }
          if constexpr (CL > 1) fence_proxy_async_acquire_peers();  // peers' rows, for the MMA
          // the correction warps' pass comes first only in a tile in which some row rescales
          // (all rows are checked: a straight run of loads measured faster than a loop over
          // the rows in use)
          bool resc = false;
          if (t > 0) {
            const float4* a4 = reinterpret_cast<const float4*>(alpha_s + s * kPRows);
#pragma unroll
            for (int i = 0; i < kPRows / 4; ++i) {
              const float4 v = a4[i];
              resc |= (v.x != 1.f) | (v.y != 1.f) | (v.z != 1.f) | (v.w != 1.f);
            }
          }
          if (resc && !mbar_wait(&corr[s], ph, p.status, p.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int r_lo = it.row0 + t * TT;
          const int nks = (min(TT, it.row1 - r_lo) + 15) / 16;
          for (int kk = 0; kk < nks; ++kk) {
            const uint64_t ad = smem_desc(pa + kk * 256, 128, (TT / 8) * 128, kLayoutNone);
            for (int c = 0; c < dS; c += 256) {
              const int hf = c >> 9, n0 = c & 511;
              const int N = min(256, dS - c);
              const uint64_t bd = smem_desc(ka + kk * slab_bytes + (c / 64) * 2048, 2048, 1024, kLayoutSW128);
              umma_f16(tmem + (static_cast<uint32_t>(16 * hf) << 16) + static_cast<uint32_t>(n0), ad, bd,
                       idesc_bf16_f32(kPRows, static_cast<uint32_t>(N), 0u, 1u), (t > 0 || kk > 0) ? 1u : 0u);
            }
          }
          umma_commit(&empty[s]);
          // pempty releases the P stage and its alphas to every writer: the correction warps
          // must have read the alphas first
          if (!resc && !mbar_wait(&corr[s], ph, p.status, p.wait_ns)) {
            ok = false;
            break;
          }
          if (CL > 1) umma_commit_mc(&pempty[s], static_cast<uint16_t>((1u << CL) - 1u));
          else umma_commit(&pempty[s]);
        }
        umma_commit(accfull);  // also after a failed tile: covers every MMA issued so far
        ++ii;
      }
      // no MMA may be in flight at teardown: wait for the last commit
      if (ii > 0) mbar_wait(accfull, static_cast<uint32_t>(ii - 1) & 1u, p.status, p.wait_ns);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ correction + epilogue warpgroup
    // Lane l of quarter q holds P row 16 q + l % 16 (head n, or padding: n < 0) in accumulator
    // half l / 16.
    const int quarter = warp & 3;
    const int prow = 16 * quarter + (lane & 15), hf = lane >> 4;
    const int n = row_head(prow, CL, H_own);
    const int hcols = min(512, dS);  // columns per accumulator half
    const int my_cols = min(512, max(dS - 512 * hf, 0));
    const uint32_t tbase = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    int g = 0, ii = 0;
    bool ok = true;
    for (; ok && cur.next(it, s_nb, s_q, s_soff); ++ii) {
      const int nt = tiles_of(it);
      for (int t = 0; t < nt; ++t, ++g) {
        const int s = g % stages;
        const uint32_t ph = static_cast<uint32_t>(g / stages) & 1u;
        if (!__all_sync(0xffffffffu, mbar_wait<(CL > 1)>(&pfull[s], ph, p.status, p.wait_ns))) {
          ok = false;
          break;
        }
        const float alpha = alpha_s[s * kPRows + prow];  // 1 in padding rows
        if (t > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
          // rescale this quarter's rows once the previous tile's MMAs have finished
          const int sp = (g - 1) % stages;
          const uint32_t php = static_cast<uint32_t>((g - 1) / stages) & 1u;
          if (!__all_sync(0xffffffffu, mbar_wait(&empty[sp], php, p.status, p.wait_ns))) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int c = 0; c < hcols; c += 16) {
            float v[16];
            tmem_ld16(tbase + c, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] *= alpha;
            tmem_st16(tbase + c, v);
          }
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&corr[s]);
      }
      if (!ok) break;
      // epilogue: accumulator rows -> partial U[slot][head][own columns]
      if (!__all_sync(0xffffffffu, mbar_wait(accfull, static_cast<uint32_t>(ii) & 1u, p.status, p.wait_ns))) break;
      tc_fence_after();
      float* dst = p.ws_U + (static_cast<size_t>(it.slot) * p.H + max(n, 0)) * p.d + col0 + 512 * hf;
      // four 16-column loads in flight per wait (hcols and my_cols are multiples of 64)
      for (int c = 0; c < hcols; c += 64) {
        float v[4][16];
#pragma unroll
        for (int j = 0; j < 4; ++j) tmem_ld16(tbase + c + 16 * j, v[j]);
        tmem_wait_ld();
        if (n >= 0 && c < my_cols) {
#pragma unroll
          for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int i = 0; i < 16; i += 4)
              *reinterpret_cast<float4*>(dst + c + 16 * j + i) =
                  make_float4(v[j][i], v[j][i + 1], v[j][i + 2], v[j][i + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(accempty);
    }
  } else {
    // ------------------------------------------------------------ score / softmax warps
    const int sw = warp - 6;
    const bool hbal = balanced_heads_fit(H_own, HPW);
    constexpr int HPP = 32 / TT;                  // heads per pass (one row per lane)
    constexpr int NPASS = (HPW + HPP - 1) / HPP;  // passes over this warp's heads
    // TT = 32: lane (chunk c = lane % 8, row group rg = lane / 8) multiplies 16-byte chunk c of
    // rows rg, rg + 4, ... by q held in registers, and a butterfly over the 8 chunk lanes leaves
    // row rg + 4 c in the lane. TT = 16: one row per lane, two heads per pass.
    const int row = TT == 32 ? (lane >> 3) + 4 * (lane & 7) : lane % TT, hslot = lane / TT;
    const uint32_t kbase = smem_u32(kst);
    const uint32_t pst_base = smem_u32(pst);
    int mrow[NPASS];  // P row of this lane's head in each pass
#pragma unroll
    for (int ps = 0; ps < NPASS; ++ps) {
      const int k = ps * HPP + hslot;
      const int hh = softmax_head(sw, k, H_own, hbal);
      mrow[ps] = (k < HPW && hh < H_own) ? p_row(head0 + hh, CL, H_own) : 0;
    }
    int g = 0;
    bool ok = true;
    while (ok && cur.next(it, s_nb, s_q, s_soff)) {
      const int nt = tiles_of(it);
      const int b = it.b;
      const int nb_old = it.nb - p.append;  // rows holding cached keys
      // q of this warp's heads to shared memory (read back as broadcasts, or kept in registers
      // for this lane's chunks when TT = 32)
      float mref[NPASS], lsum[NPASS];  // running max and sum of this lane's head in each pass
      uint64_t qp[TT == 32 ? HPW : 1][DHB][4];  // q pairs of this lane's chunk (fma.rn.f32x2 operands)
#pragma unroll
      for (int ps = 0; ps < NPASS; ++ps) {
        mref[ps] = -INFINITY;
        lsum[ps] = 0.f;
      }
      __syncwarp();
#pragma unroll
      for (int k = 0; k < HPW; ++k) {
        const int hh = softmax_head(sw, k, H_own, hbal);
        if (hh < H_own) {
          const float* src = p.q + static_cast<size_t>(b) * p.d + col0 + hh * DH;
          for (int i = lane; i < DH / 4; i += 32)
            reinterpret_cast<float4*>(q_s + hh * DH)[i] = __ldg(reinterpret_cast<const float4*>(src) + i);
        }
      }
      __syncwarp();
      if constexpr (TT == 32) {
#pragma unroll
        for (int k = 0; k < HPW; ++k) {
          const int hh = softmax_head(sw, k, H_own, hbal);
#pragma unroll
          for (int jj = 0; jj < DHB; ++jj) {
            const float4* qv = reinterpret_cast<const float4*>(q_s + (hh < H_own ? hh : 0) * DH + 8 * ((lane & 7) + 8 * jj));
            const float4 qa = qv[0], qb = qv[1];
            qp[k][jj][0] = pack2(qa.x, qa.y);
            qp[k][jj][1] = pack2(qa.z, qa.w);
            qp[k][jj][2] = pack2(qb.x, qb.y);
            qp[k][jj][3] = pack2(qb.z, qb.w);
          }
        }
      }

      for (int t = 0; t < nt; ++t, ++g) {
        const int s = g % stages;
        const uint32_t ph = static_cast<uint32_t>(g / stages) & 1u;
        const int r_lo = it.row0 + t * TT;
        const int nvalid = min(TT, it.row1 - r_lo);
        const int nloaded = (nvalid + 15) & ~15;
        if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph, p.status, p.wait_ns))) {
          ok = false;
          break;
        }
        uint8_t* ks_ptr = kst + s * kstage_bytes;

        // Rows >= nb_old in this tile hold no cached key: the appended key goes
        // to row nb_old (also written to the cache), the rest become zero. Each
        // warp fixes the column blocks of its own heads; the MMA reads them
        // after the proxy fence and the pfull/corr barriers below.
        if (r_lo + nloaded > nb_old) {
          const int fr0 = max(nb_old - r_lo, 0);
#pragma unroll
          for (int k = 0; k < HPW; ++k) {
            const int hh = softmax_head(sw, k, H_own, hbal);
            if (hh >= H_own) continue;
#pragma unroll
            for (int c = 0; c < DHB; ++c) {
              const int cb = hh * DHB + c;
              for (int i = lane; i < (nloaded - fr0) * 8; i += 32) {
                const int rw = fr0 + (i >> 3), j = i & 7;
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (p.append && r_lo + rw == nb_old) {
                  const size_t col = static_cast<size_t>(col0) + cb * 64 + j * 8;
                  v = __ldg(reinterpret_cast<const uint4*>(p.k_new + static_cast<size_t>(b) * p.d + col));
                  *reinterpret_cast<uint4*>(p.kcache + (static_cast<size_t>(b) * p.cap + nb_old) * p.d + col) = v;
                }
                *reinterpret_cast<uint4*>(ks_ptr + (rw >> 4) * slab_bytes + cb * 2048 + (rw & 15) * 128 +
                                          ((j ^ (rw & 7)) << 4)) = v;
              }
            }
          }
          __syncwarp();
        }

        // P stage s is free once every CTA's MMAs and copies of tile g - stages finished with
        // it and its correction warps read the alphas (each MMA thread commits after both).
        if (g >= stages && !__all_sync(0xffffffffu, mbar_wait<(CL > 1)>(&pempty[s], ph ^ 1u, p.status, p.wait_ns))) {
          ok = false;
          break;
        }

        const uint32_t kt = kbase + s * kstage_bytes;
        // Phase 1: scores on the CUDA cores (the tensor pipe is left to the P·K MMAs), fp32
        // accumulation, K read once from the swizzled stage with conflict-free 16-byte loads.
        float sc[NPASS];
        if constexpr (TT == 32) {
          const int c = lane & 7, rg = lane >> 3;
#pragma unroll
          for (int k = 0; k < HPW; ++k) {
            const int hh = softmax_head(sw, k, H_own, hbal);
            sc[k] = -INFINITY;
            if (hh >= H_own) continue;  // warp-uniform: this warp has no head in slot k
            float pr[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int r = rg + 4 * i;
              const uint32_t rbase = kt + (r >> 4) * slab_bytes + (r & 15) * 128;
              // even columns accumulate in the low half, odd columns in the high half
              uint64_t acc = pack2(0.f, 0.f);
#pragma unroll
              for (int jj = 0; jj < DHB; ++jj) {
                const int colk = hh * DH + 8 * (c + 8 * jj);
                uint4 kv;
                asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(kv.x), "=r"(kv.y), "=r"(kv.z), "=r"(kv.w)
                             : "r"(rbase + (colk >> 6) * 2048 + ((((colk & 63) >> 3) ^ (r & 7)) << 4)));
                acc = ffma2(pack2(bf16lo(kv.x), bf16hi(kv.x)), qp[k][jj][0], acc);
                acc = ffma2(pack2(bf16lo(kv.y), bf16hi(kv.y)), qp[k][jj][1], acc);
                acc = ffma2(pack2(bf16lo(kv.z), bf16hi(kv.z)), qp[k][jj][2], acc);
                acc = ffma2(pack2(bf16lo(kv.w), bf16hi(kv.w)), qp[k][jj][3], acc);
              }
              pr[i] = unpack_sum(acc);
            }
            // butterfly over the chunk lanes: after the level with mask m each lane keeps the
            // rows whose index bit (m) matches its own chunk bit, summed over both lanes
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const bool up = c & 4;
              const float recv = __shfl_xor_sync(0xffffffffu, up ? pr[i] : pr[i + 4], 4);
              pr[i] = (up ? pr[i + 4] : pr[i]) + recv;
            }
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const bool up = c & 2;
              const float recv = __shfl_xor_sync(0xffffffffu, up ? pr[i] : pr[i + 2], 2);
              pr[i] = (up ? pr[i + 2] : pr[i]) + recv;
            }
            {
              const bool up = c & 1;
              const float recv = __shfl_xor_sync(0xffffffffu, up ? pr[0] : pr[1], 1);
              pr[0] = (up ? pr[1] : pr[0]) + recv;
            }
            sc[k] = row < nvalid ? pr[0] * p.scale_log2 : -INFINITY;
          }
        } else {
#pragma unroll
          for (int ps = 0; ps < NPASS; ++ps) {
            const int k = ps * HPP + hslot;
            const int hh = softmax_head(sw, k, H_own, hbal);
            float a0 = 0.f, a1 = 0.f;
            if (k < HPW && hh < H_own) {
              const uint32_t rbase = kt + (row >> 4) * slab_bytes + (row & 15) * 128;
              const float4* qv = reinterpret_cast<const float4*>(q_s + hh * DH);
#pragma unroll
              for (int j = 0; j < DH / 8; ++j) {
                const int colk = hh * DH + 8 * j;
                uint4 kv;
                asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(kv.x), "=r"(kv.y), "=r"(kv.z), "=r"(kv.w)
                             : "r"(rbase + (colk >> 6) * 2048 + ((((colk & 63) >> 3) ^ (row & 7)) << 4)));
                const float4 qa = qv[2 * j], qb = qv[2 * j + 1];
                a0 = fmaf(bf16lo(kv.x), qa.x, a0);
                a1 = fmaf(bf16hi(kv.x), qa.y, a1);
                a0 = fmaf(bf16lo(kv.y), qa.z, a0);
                a1 = fmaf(bf16hi(kv.y), qa.w, a1);
                a0 = fmaf(bf16lo(kv.z), qb.x, a0);
                a1 = fmaf(bf16hi(kv.z), qb.y, a1);
                a0 = fmaf(bf16lo(kv.w), qb.z, a0);
                a1 = fmaf(bf16hi(kv.w), qb.w, a1);
              }
            }
            sc[ps] = (k < HPW && hh < H_own && row < nvalid) ? (a0 + a1) * p.scale_log2 : -INFINITY;
          }
        }
        // Phase 2: tile maxima (over the TT lanes of a head)
        float mx[NPASS];
#pragma unroll
        for (int ps = 0; ps < NPASS; ++ps) mx[ps] = sc[ps];
#pragma unroll
        for (int o = TT / 2; o > 0; o >>= 1)
#pragma unroll
          for (int ps = 0; ps < NPASS; ++ps) mx[ps] = fmaxf(mx[ps], __shfl_xor_sync(0xffffffffu, mx[ps], o));
        // Phase 3: lazy running max, P and alpha to this CTA's rows of the stage
#pragma unroll
        for (int ps = 0; ps < NPASS; ++ps) {
          const int k = ps * HPP + hslot;
          const int hh = softmax_head(sw, k, H_own, hbal);
          if (k >= HPW || hh >= H_own) continue;
          float alpha = 1.f;
          if (t == 0) {
            mref[ps] = mx[ps];
          } else if (mx[ps] > mref[ps] + kLazyRescaleLog2) {
            alpha = exp2f(mref[ps] - mx[ps]);
            mref[ps] = mx[ps];
            lsum[ps] *= alpha;
          }
          const int m = mrow[ps];
          const float pv = row < nvalid ? exp2f(sc[ps] - mref[ps]) : 0.f;
          const __nv_bfloat16 pb = __float2bfloat16_rn(pv);
          lsum[ps] += __bfloat162float(pb);
          const uint32_t off = static_cast<uint32_t>(s) * pstage_bytes +
                               static_cast<uint32_t>(((m >> 3) * (TT / 8) + (row >> 3)) * 128 + (m & 7) * 16 + (row & 7) * 2);
          const uint16_t bits = __bfloat16_as_ushort(pb);
          asm volatile("st.shared.u16 [%0], %1;" ::"r"(pst_base + off), "h"(bits) : "memory");
          if (row == 0) alpha_s[s * kPRows + m] = alpha;
        }
        // the MMA operand reads P through the async proxy
        fence_proxy_async_smem();
        if constexpr (CL > 1) {
          // every peer gets this warp's rows of P (16-byte chunks of 8 rows) and alphas by
          // stores that complete on the peer's pfull
          __syncwarp();
          constexpr int kChunks = HPW * (TT / 8);
          if (lane < kChunks || lane >= 32 - HPW) {
            const int k = lane < kChunks ? lane / (TT / 8) : 31 - lane;
            const int hh = softmax_head(sw, k, H_own, hbal);
            if (hh < H_own) {
              const int m = p_row(head0 + hh, CL, H_own);
              const uint32_t bar = smem_u32(&pfull[s]);
              if (lane < kChunks) {
                const uint32_t off = static_cast<uint32_t>(s) * pstage_bytes +
                                     static_cast<uint32_t>(((m >> 3) * (TT / 8) + lane % (TT / 8)) * 128 + (m & 7) * 16);
                uint4 v;
                asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                             : "r"(pst_base + off));
#pragma unroll
                for (int r = 1; r < CL; ++r) {
                  const uint32_t peer = (rank + r) % CL;
                  st_async_v4(mapa_shared(pst_base + off, peer), v, mapa_shared(bar, peer));
                }
              } else {
                const uint32_t a = smem_u32(alpha_s + s * kPRows + m);
                const uint32_t v = __float_as_uint(alpha_s[s * kPRows + m]);
#pragma unroll
                for (int r = 1; r < CL; ++r) {
                  const uint32_t peer = (rank + r) % CL;
                  st_async_b32(mapa_shared(a, peer), v, mapa_shared(bar, peer));
                }
              }
            }
          }
        }
        __syncwarp();
        if (lane == 0) {
          // the peers' rows arrive as transaction bytes: H_own heads x (TT P values + alpha) each
          if (CL > 1 && sw == 0)
            mbar_arrive_expect_tx(&pfull[s], static_cast<uint32_t>((CL - 1) * H_own * (TT * 2 + 4)));
          else
            mbar_arrive(&pfull[s]);
        }
      }
      if (!ok) break;
      const size_t slot = static_cast<size_t>(it.slot);
#pragma unroll
      for (int ps = 0; ps < NPASS; ++ps) {
        const int k = ps * HPP + hslot;
        const int hh = softmax_head(sw, k, H_own, hbal);
        float tot = lsum[ps];
#pragma unroll
        for (int o = TT / 2; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
        if (k < HPW && hh < H_own && row == 0) {
          p.ws_m[slot * p.H + head0 + hh] = mref[ps];
          p.ws_l[slot * p.H + head0 + hh] = tot;
        }
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  // Reconverge every warp first: in the producer and MMA warps only lane 0 ran
  // the loop, and a CTA barrier reached by a split warp does not wait for it.
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, p.tmem_cols);
  }
  if (CL > 1) cluster_sync();
}

// ---------------------------------------------------------------------------- host side
namespace {

struct TCConfig {
  int CL, TT, DHB, HPW, stages;
  uint32_t tmem_cols, smem;
};

// Template instances compiled below (CL, TT, DHB, HPW); pick_config only returns these.
#define SLIM_TC_INSTANCES(X)                                                                               \
  X(1, 32, 1, 1) X(1, 32, 1, 2) X(1, 32, 1, 3) X(1, 32, 1, 4) X(1, 32, 2, 1) X(1, 32, 2, 2) X(2, 32, 1, 1) \
  X(2, 32, 1, 2) X(2, 32, 1, 3) X(2, 32, 1, 4) X(2, 32, 2, 1) X(2, 32, 2, 2) X(4, 32, 1, 1) X(4, 32, 1, 2) \
  X(4, 32, 2, 1) X(4, 32, 2, 2) X(1, 16, 1, 1) X(1, 16, 1, 2) X(1, 16, 1, 3) X(1, 16, 1, 4) X(1, 16, 2, 1) \
  X(1, 16, 2, 2) X(2, 16, 1, 1) X(2, 16, 1, 2) X(2, 16, 1, 3) X(2, 16, 1, 4) X(2, 16, 2, 1) X(2, 16, 2, 2) \
  X(4, 16, 1, 1) X(4, 16, 1, 2) X(4, 16, 2, 1) X(4, 16, 2, 2)

bool tc_instantiated(int CL, int TT, int DHB, int HPW) {
#define SLIM_TC_MATCH(a, b, c, e) \
  if (CL == a && TT == b && DHB == c && HPW == e) return true;
  SLIM_TC_INSTANCES(SLIM_TC_MATCH)
#undef SLIM_TC_MATCH
  return false;
}

uint32_t pow2_cols(uint32_t c) {
  uint32_t r = 32;
  while (r < c) r <<= 1;
  return r;
}

// SLIM_SPLIT_CLUSTER=1|2|4 in the environment forces the cluster size of the
// split kernel where that size is valid for the shape (a tuning knob; read once).
int forced_cluster() {
  static const int v = [] {
    const char* e = std::getenv("SLIM_SPLIT_CLUSTER");
    const int c = e ? std::atoi(e) : 0;
    return (c == 1 || c == 2 || c == 4) ? c : 0;
  }();
  return v;
}

bool pick_config(int B, int d, int H, TCConfig* out) {
  if (H <= 0 || d % H || H > kPRows) return false;
  const int dh = d / H;
  if (dh != 64 && dh != 128) return false;
  const int smem_cap = max_smem_optin();
  const int force = forced_cluster();
  for (int pass = force ? 0 : 1; pass < 2; ++pass)
  for (int CL = 1; CL <= 4; CL *= 2) {
    if (pass == 0 && CL != force) continue;
    if (d % (64 * CL) || H % CL || (d / CL) % dh || d / CL > kMaxColsPerCTA) continue;
    const int H_own = H / CL;
    const int HPW = (H_own + kSoftmaxWarps - 1) / kSoftmaxWarps;
    for (int TT : {32, 16}) {
      int stages = 0;
      for (int s = 8; s >= 2; --s) {
        if (tc_smem_layout(CL, TT, d, s, B).total <= static_cast<uint32_t>(smem_cap)) {
          stages = s;
          break;
        }
      }
      if (stages < (TT == 32 ? 3 : 2)) continue;
      if (!tc_instantiated(CL, TT, dh / 64, HPW)) continue;
      out->CL = CL;
      out->TT = TT;
      out->DHB = dh / 64;
      out->HPW = HPW;
      out->stages = stages;
      out->tmem_cols = pow2_cols(static_cast<uint32_t>(std::min(d / CL, 512)));
      out->smem = tc_smem_layout(CL, TT, d, stages, B).total;
      return true;
    }
  }
  return false;
}

// Clusters of CL CTAs that can be resident at once. A cluster must fit in one
// GPC, so with CL > 1 fewer than num_sms / CL clusters may fit; launching more
// would run the extra ones as a second wave. Memoised per (device, smem).
template <int CL, int TT, int DHB, int HPW>
int resident_clusters(cudaLaunchConfig_t cfg) {
  static std::mutex mu;
  static std::map<std::pair<int, uint32_t>, int> memo;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  const std::pair<int, uint32_t> key(dev, static_cast<uint32_t>(cfg.dynamicSmemBytes));
  std::lock_guard<std::mutex> lock(mu);
  auto it = memo.find(key);
  if (it != memo.end()) return it->second;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, decode_b_tc_kernel<CL, TT, DHB, HPW>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  memo[key] = n;
  return n;
}

template <int CL, int TT, int DHB, int HPW>
cudaError_t launch_tc(const CUtensorMap& map, DecodeTCParams prm, const TCConfig& c, cudaStream_t st) {
  auto kern = decode_b_tc_kernel<CL, TT, DHB, HPW>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(c.smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(prm.n_groups * CL), 1, 1);
  cfg.blockDim = dim3(kTCThreads, 1, 1);
  cfg.dynamicSmemBytes = c.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  if (CL > 1) {
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const int fit = resident_clusters<CL, TT, DHB, HPW>(cfg);
    if (fit > 0 && fit < prm.n_groups) {
      prm.n_groups = fit;
      cfg.gridDim = dim3(static_cast<unsigned>(fit * CL), 1, 1);
    }
    cfg.numAttrs = 2;
  } else {
    cfg.attrs = attr + 1;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, kern, map, prm);
}

}  // namespace

bool decode_b_tc_supported(int B, int d, int H) {
  TCConfig c;
  return pick_config(B, d, H, &c);
}

int decode_b_tc_cluster(int B, int d, int H) {
  TCConfig c;
  return pick_config(B, d, H, &c) ? c.CL : 0;
}

cudaError_t launch_decode_b_tc(const DecodeArgs& a, const SplitWorkspace& ws, cudaStream_t st, int* launches) {
  TCConfig c;
  if (a.dtype != SLIM_BF16 || !pick_config(a.B, a.d, a.H, &c)) return cudaErrorNotSupported;
  CUtensorMap map;
  // K cache viewed as [d/64 column blocks][B*cap rows][64 columns]; a box is 64 x 16 x (d/CL/64)
  if (!encode_tmap_kslab(&map, a.kcache, static_cast<uint64_t>(a.B) * a.cap, a.d, a.d / c.CL / 64))
    return cudaErrorInvalidValue;
  DecodeTCParams prm;
  prm.q = a.q;
  prm.k_new = static_cast<const __nv_bfloat16*>(a.k_new);
  prm.kcache = static_cast<__nv_bfloat16*>(a.kcache);
  prm.lens = a.lens;
  prm.status = a.status;
  prm.ws_U = ws.U;
  prm.ws_m = ws.m;
  prm.ws_l = ws.l;
  prm.ws_meta = ws.meta;
  prm.B = a.B;
  prm.d = a.d;
  prm.H = a.H;
  prm.cap = a.cap;
  prm.append = a.k_new != nullptr ? 1 : 0;
  prm.n_groups = num_sms() / c.CL;
  prm.stages = c.stages;
  prm.min_rows = max(16, 8 * a.H);
  prm.tmem_cols = c.tmem_cols;
  prm.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(a.d / a.H));
  prm.wait_ns = a.wait_ns ? a.wait_ns : kWaitLimitNs;
  prm.stall = a.stall;
  cudaError_t e = cudaErrorNotSupported;
#define SLIM_TC_CASE(CL_, TT_, DHB_, HPW_)                           \
  if (c.CL == CL_ && c.TT == TT_ && c.DHB == DHB_ && c.HPW == HPW_) { \
    e = launch_tc<CL_, TT_, DHB_, HPW_>(map, prm, c, st);             \
  } else
  SLIM_TC_INSTANCES(SLIM_TC_CASE) { e = cudaErrorNotSupported; }
#undef SLIM_TC_CASE
  if (e == cudaSuccess && launches) ++*launches;
  return e;
}

}  // namespace slim
