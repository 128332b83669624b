// Generation step, ordering (a), on tensor cores (bf16 K cache, d % 256 == 0,
// d_h = 64 or 128).
//
// Slim Attention article, section "K-Cache is All You Need", generation phase,
// first option: compute the values V = K·W_KV from the cached keys, then
// multiply the softmax rows by V. Here V is computed one tile at a time and
// used where it is made: a tile is 128 attended rows of one sequence x 256
// columns of V (a group of 4 heads at d_h = 64, 2 at d_h = 128), so
//     V_tile = K[rows, :] · W_KV[:, tile columns]      (tcgen05, fp32 in TMEM)
//     o_h   += Σ_t p_ht V_tile[t, h-cols]              (epilogue, CUDA cores)
// and V never reaches global memory. Per tile the partial of every head of the
// group is (m_h, l_h, o_h) with the max and sum taken over the tile's rows; a
// merge kernel combines the row tiles of a sequence by the log-sum-exp rule.
//
// Persistent CTAs (one per SM) walk the tiles, tile index = (row tile of all
// sequences) x (column groups) + column group, which is also the partial slot.
// Per CTA (10 warps):
//   warp 0      TMA producer: per 64-column chunk k, the K rows (128 x 64,
//               K-major, 128-byte swizzle) and W_KV[64 k .., tile columns]
//               (64 x 256, MN-major) into a 4-stage ring;
//   warp 1      MMA issuer: tcgen05.mma M=128 N=256 K=16 into one of two TMEM
//               accumulators (512 columns), so a tile's epilogue overlaps the
//               next tile's main loop;
//   warps 2..5  epilogue: row t of the accumulator in lane t, p_ht = 2^(s_ht -
//               m_h) applied per column, rows summed by a butterfly over the
//               warp and the four warps' sums added in shared memory;
//   warps 6..9  scores: row t in lane t; s_ht = q_h·K_t/sqrt(d_h) from the
//               K chunks of the tile's heads while they are in shared memory.
// Rows past a sequence's attended length (the tile's tail) get p = 0 and are
// left out of the sums. Every wait is bounded (SLIM_DEV_TIMEOUT); a CTA that
// gives up drains its copies and MMAs and frees TMEM before it exits.
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace slim {

namespace {

constexpr int kABM = 128, kABN = 256, kABK = 64, kAStages = 4;
constexpr int kAThreads = 10 * 32;
constexpr uint32_t kAStageA = kABM * kABK * 2;  // 16 KB
constexpr uint32_t kAStageB = kABK * kABN * 2;  // 32 KB

struct DecodeATCParams {
  const float* q;
  const int32_t* lens;
  int32_t* status;
  float* ws_O;      // [tiles][256] unnormalised p·V of the tile's columns
  float* ws_m;      // [tiles][4] max over the tile's rows (log2 domain), per head of the group
  float* ws_l;      // [tiles][4]
  int32_t* ws_meta; // [1 + b]: first row tile of sequence b (b = 0..B); [2 + B + b]: flags
  int B, d, H;
  int64_t cap;
  int append;       // this step's k is already at row lens[b]; attend over lens[b] + 1 rows
  float scale_log2;
};

struct ATCSmem {
  uint32_t a, b, sc, qs, red, redml, bars, slot, plan, total;
};
__host__ __device__ inline ATCSmem atc_smem_layout(int B) {
  ATCSmem s;
  uint32_t o = 0;
  s.a = o;
  o += kAStages * kAStageA;
  s.b = o;
  o += kAStages * kAStageB;
  s.sc = o;  // [2 accumulators][128 rows][4 heads] scaled scores
  o += 2u * kABM * 4u * 4u;
  s.qs = o;  // [256] q of the tile's columns
  o += kABN * 4u;
  s.red = o;  // [4 warps][256] column sums
  o += 4u * kABN * 4u;
  s.redml = o;  // [4 warps][4 heads] max, then sums
  o += 2u * 4u * 4u * 4u;
  s.bars = o;  // full, empty per stage; accfull, accempty, scready per accumulator
  o += (2u * kAStages + 6u) * 8u;
  s.slot = o;
  o += 16u;
  s.plan = o;  // s_nb [B], s_rtb [B + 1]
  o += (2u * static_cast<uint32_t>(B) + 2u) * 4u;
  s.total = o + 1024u;
  return s;
}

__global__ void __launch_bounds__(kAThreads, 1)
    decode_a_tc_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap wmap,
                       const DecodeATCParams p) {
  extern __shared__ uint8_t asm_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(asm_raw) + 1023) & ~uintptr_t(1023));
  const ATCSmem L = atc_smem_layout(p.B);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* as = sm + L.a;
  uint8_t* bs = sm + L.b;
  float* sc = reinterpret_cast<float*>(sm + L.sc);
  float* q_s = reinterpret_cast<float*>(sm + L.qs);
  float* red = reinterpret_cast<float*>(sm + L.red);
  float* redml = reinterpret_cast<float*>(sm + L.redml);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L.bars);
  uint64_t* empty = full + kAStages;
  uint64_t* accfull = empty + kAStages;  // [2]
  uint64_t* accempty = accfull + 2;      // [2]
  uint64_t* scready = accempty + 2;      // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L.slot);
  int* s_nb = reinterpret_cast<int*>(sm + L.plan);
  int* s_rtb = s_nb + p.B;
  const int d = p.d, dh = d / p.H, CT = d / kABN, nk = d / kABK;

  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&wmap);
  } else if (warp == 1) {
    if (lane == 0) {
      for (int s = 0; s < kAStages; ++s) {
        mbar_init(&full[s], 1);
        mbar_init(&empty[s], 1 + 4);  // the MMAs' commit and the four score warps
      }
      for (int a = 0; a < 2; ++a) {
        mbar_init(&accfull[a], 1);
        mbar_init(&accempty[a], 4);
        mbar_init(&scready[a], 4);
      }
      fence_barrier_init();
    }
    __syncwarp();
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  pdl_wait_primary();
  pdl_launch_dependents();
  if (warp == 0) {
    // row tiles of every sequence; length errors reported once (CTA 0)
    int bad = 0;
    for (int b = lane; b < p.B; b += 32) {
      const int Lb = __ldcg(p.lens + b);
      int nb;
      if (Lb < 0 || static_cast<int64_t>(Lb) > p.cap) {
        nb = 0;
        bad |= SLIM_DEV_BADLEN;
      } else if (p.append && static_cast<int64_t>(Lb) >= p.cap) {
        nb = 0;
        bad |= SLIM_DEV_OVERFLOW;
      } else {
        nb = Lb + p.append;
      }
      s_nb[b] = nb;
      if (blockIdx.x == 0) p.ws_meta[2 + p.B + b] = (nb > 0 && p.append) ? kSeqAppend : 0;
    }
    bad = __reduce_or_sync(0xffffffffu, bad);
    if (blockIdx.x == 0 && lane == 0 && bad) atomicOr(p.status, bad);
    __syncwarp();
    int carry = 0;
    for (int base = 0; base < p.B; base += 32) {
      const int b = base + lane;
      const int c = b < p.B ? (s_nb[b] + kABM - 1) / kABM : 0;
      int x = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (b < p.B) s_rtb[b] = carry + x - c;
      carry += __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) s_rtb[p.B] = carry;
    __syncwarp();
    if (blockIdx.x == 0)
      for (int b = lane; b <= p.B; b += 32) p.ws_meta[1 + b] = s_rtb[b];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_tiles = s_rtb[p.B] * CT;
  // tile -> (sequence, first row, rows, column group)
  auto tile_of = [&](int tau, int& b, int& r0, int& nv, int& ct) {
    const int rt = tau / CT;
    ct = tau - rt * CT;
    int lo = 0, hi = p.B;  // largest b with s_rtb[b] <= rt
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s_rtb[mid] <= rt) lo = mid; else hi = mid;
    }
    b = lo;
    while (b + 1 < p.B && s_rtb[b + 1] <= rt) ++b;  // skip sequences without tiles
    r0 = (rt - s_rtb[b]) * kABM;
    nv = min(kABM, s_nb[b] - r0);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_a = l2_policy_evict_first(), pol_w = l2_policy_evict_last();
      int g = 0;
      bool ok = true;
      for (int tau = blockIdx.x; tau < n_tiles && ok; tau += gridDim.x) {
        int b, r0, nv, ct;
        tile_of(tau, b, r0, nv, ct);
        const int y = static_cast<int>(static_cast<int64_t>(b) * p.cap + r0);
        for (int k = 0; k < nk; ++k, ++g) {
          const int s = g % kAStages;
          const uint32_t ph = static_cast<uint32_t>(g / kAStages) & 1u;
          if (g >= kAStages && !mbar_wait(&empty[s], ph ^ 1u, p.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], kAStageA + kAStageB);
          tma_load_2d(as + s * kAStageA, &kmap, k * kABK, y, &full[s], pol_a);
          tma_load_3d(bs + s * kAStageB, &wmap, 0, k * kABK, ct * (kABN / 64), &full[s], pol_w);
        }
      }
      for (int t = max(0, g - kAStages); t < g; ++t)  // every issued copy lands before exit
        mbar_wait(&full[t % kAStages], static_cast<uint32_t>(t / kAStages) & 1u, p.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kABM, kABN, 0u, 1u);
      const uint32_t abase = smem_u32(as), bbase = smem_u32(bs);
      int g = 0, i = 0;
      bool ok = true;
      for (int tau = blockIdx.x; tau < n_tiles && ok; tau += gridDim.x, ++i) {
        const int ab = i & 1;
        // the epilogue of tile i - 2 must have read this accumulator
        if (i >= 2 && !mbar_wait(&accempty[ab], static_cast<uint32_t>((i - 2) >> 1) & 1u, p.status)) break;
        tc_fence_after();
        const uint32_t acc = tmem + static_cast<uint32_t>(ab * kABN);
        for (int k = 0; k < nk; ++k, ++g) {
          const int s = g % kAStages;
          const uint32_t ph = static_cast<uint32_t>(g / kAStages) & 1u;
          if (!mbar_wait(&full[s], ph, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kABK / 16; ++kk) {
            // A: K-major, 128-byte swizzle, 8-row groups 1024 B apart; a 16-column step is 32 B.
            const uint64_t ad = smem_desc(abase + s * kAStageA + kk * 32, 16, 1024, kLayoutSW128);
            // B: MN-major, 64-column blocks 64 rows x 128 B (8 KB) apart, 8-row groups 1024 B apart.
            const uint64_t bd = smem_desc(bbase + s * kAStageB + kk * 16 * 128, kABK * 128, 1024, kLayoutSW128);
            umma_f16(acc, ad, bd, idesc, (k > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty[s]);
        }
        umma_commit(&accfull[ab]);  // also after a failed chunk: covers every MMA issued so far
        if (!ok) {
          ++i;
          break;
        }
      }
      if (i > 0) mbar_wait(&accfull[(i - 1) & 1], static_cast<uint32_t>((i - 1) >> 1) & 1u, p.status);
    }
  } else if (warp >= 6) {
    // ------------------------------------------------------------ scores
    const int t = (warp - 6) * 32 + lane;  // row of the tile
    const uint32_t abase = smem_u32(as);
    int g = 0, i = 0;
    bool ok = true;  // the four score warps stop together (their named barriers stay aligned)
    for (int tau = blockIdx.x; tau < n_tiles && ok; tau += gridDim.x, ++i) {
      const int ab = i & 1;
      int b, r0, nv, ct;
      tile_of(tau, b, r0, nv, ct);
      // q of the tile's columns; the previous tile's readers are past the barrier below
      named_barrier_sync(1, 128);
      for (int c = (warp - 6) * 32 + lane; c < kABN; c += 128) q_s[c] = __ldg(p.q + static_cast<size_t>(b) * d + ct * kABN + c);
      named_barrier_sync(1, 128);
      float s4[4] = {0.f, 0.f, 0.f, 0.f};
      bool tile_ok = true;
      for (int k = 0; k < nk && tile_ok; ++k, ++g) {
        const int s = g % kAStages;
        const uint32_t ph = static_cast<uint32_t>(g / kAStages) & 1u;
        if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph, p.status))) {
          tile_ok = false;
          break;
        }
        const int c0 = k * kABK - ct * kABN;  // first column of the chunk within the tile
        if (c0 >= 0 && c0 < kABN) {
          const int j = c0 / dh;
          const uint32_t rowa = abase + s * kAStageA + t * 128;
          float a0 = 0.f, a1 = 0.f;
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            uint4 kv;
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(kv.x), "=r"(kv.y), "=r"(kv.z), "=r"(kv.w)
                         : "r"(rowa + ((static_cast<uint32_t>(ch ^ (t & 7))) << 4)));
            const float4 qa = *reinterpret_cast<const float4*>(q_s + c0 + ch * 8);
            const float4 qb = *reinterpret_cast<const float4*>(q_s + c0 + ch * 8 + 4);
            a0 = fmaf(bf16lo(kv.x), qa.x, a0);
            a1 = fmaf(bf16hi(kv.x), qa.y, a1);
            a0 = fmaf(bf16lo(kv.y), qa.z, a0);
            a1 = fmaf(bf16hi(kv.y), qa.w, a1);
            a0 = fmaf(bf16lo(kv.z), qb.x, a0);
            a1 = fmaf(bf16hi(kv.z), qb.y, a1);
            a0 = fmaf(bf16lo(kv.w), qb.z, a0);
            a1 = fmaf(bf16hi(kv.w), qb.w, a1);
          }
#pragma unroll
          for (int jj = 0; jj < 4; ++jj)
            if (jj == j) s4[jj] += a0 + a1;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
      // the epilogue of tile i - 2 must be done with this score buffer
      if (tile_ok && i >= 2)
        tile_ok = __all_sync(0xffffffffu,
                             mbar_wait(&accempty[ab], static_cast<uint32_t>((i - 2) >> 1) & 1u, p.status));
      ok = named_barrier_and(1, 128, tile_ok);
      if (!ok) break;
      *reinterpret_cast<float4*>(sc + (ab * kABM + t) * 4) =
          make_float4(s4[0] * p.scale_log2, s4[1] * p.scale_log2, s4[2] * p.scale_log2, s4[3] * p.scale_log2);
      __syncwarp();
      if (lane == 0) mbar_arrive(&scready[ab]);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5)
    const int quarter = warp & 3;
    const int t = quarter * 32 + lane;  // row of the tile = TMEM lane
    const int ew = warp - 2;            // index among the epilogue warps
    const int nh = kABN / dh;           // heads of the group
    int i = 0;
    for (int tau = blockIdx.x; tau < n_tiles; tau += gridDim.x, ++i) {
      const int ab = i & 1;
      const uint32_t ph = static_cast<uint32_t>(i >> 1) & 1u;
      int b, r0, nv, ct;
      tile_of(tau, b, r0, nv, ct);
      const bool got = mbar_wait(&accfull[ab], ph, p.status) && mbar_wait(&scready[ab], ph, p.status);
      if (!named_barrier_and(2, 128, got)) break;  // the four epilogue warps stop together
      tc_fence_after();
      const bool valid = t < nv;
      const float4 s = *reinterpret_cast<const float4*>(sc + (ab * kABM + t) * 4);
      const float sv[4] = {s.x, s.y, s.z, s.w};
      float mj[4], pj[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        mj[j] = warp_max(valid && j < nh ? sv[j] : -INFINITY);
        if (lane == 0) redml[ew * 4 + j] = mj[j];
      }
      named_barrier_sync(2, 128);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float m = redml[j];
#pragma unroll
        for (int w = 1; w < 4; ++w) m = fmaxf(m, redml[w * 4 + j]);
        mj[j] = m;
        pj[j] = (valid && j < nh) ? exp2f(sv[j] - m) : 0.f;
        const float ls = warp_sum(pj[j]);
        if (lane == 0) redml[16 + ew * 4 + j] = ls;
      }
      // o_c = Σ_rows p_t,h(c) V[t, c]: 16 columns at a time, summed over the warp's 32 rows
      const uint32_t tacc = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(ab * kABN);
      for (int c0 = 0; c0 < kABN; c0 += 16) {
        float v[16];
        tmem_ld16(tacc + c0, v);
        tmem_wait_ld();
        const float pw = pj[c0 / dh];
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] = valid ? pw * v[e] : 0.f;
        // butterfly reduce-scatter: after offset o a lane keeps the half selected by lane bit o
#pragma unroll
        for (int n = 16, o = 16; n >= 2; n >>= 1, o >>= 1) {
          const bool up = (lane & o) != 0;
#pragma unroll
          for (int e = 0; e < n / 2; ++e) {
            const float send = up ? v[e] : v[e + n / 2];
            const float keep = up ? v[e + n / 2] : v[e];
            v[e] = keep + __shfl_xor_sync(0xffffffffu, send, o);
          }
        }
        v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
        if ((lane & 1) == 0) red[ew * kABN + c0 + (lane >> 1)] = v[0];
      }
      tc_fence_before();
      named_barrier_sync(2, 128);  // column sums and head sums of all four warps in place
      if (lane == 0) mbar_arrive(&accempty[ab]);
      const int e0 = ew * 32 + lane;  // 128 threads, two columns each
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int c = e0 + 128 * u;
        p.ws_O[static_cast<size_t>(tau) * kABN + c] =
            red[c] + red[kABN + c] + red[2 * kABN + c] + red[3 * kABN + c];
      }
      if (e0 < 4) {
        const int j = e0;
        float m = redml[j], l = 0.f;
#pragma unroll
        for (int w = 1; w < 4; ++w) m = fmaxf(m, redml[w * 4 + j]);
#pragma unroll
        for (int w = 0; w < 4; ++w) l += redml[16 + w * 4 + j];
        p.ws_m[static_cast<size_t>(tau) * 4 + j] = m;
        p.ws_l[static_cast<size_t>(tau) * 4 + j] = l;
      }
      named_barrier_sync(2, 128);  // red and redml are reused by the next tile
    }
  }

  // ---------------------------------------------------------------- teardown
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Merge of the row tiles: out[b, ct·256 + c] = Σ_rt 2^(m - M) O[c] / Σ_rt 2^(m - M) l over the tiles of
// sequence b and column group ct; one CTA per (sequence, column group), one thread per column. The
// lengths advance here, after the tile kernel has read them.
__global__ void __launch_bounds__(kABN) merge_a_kernel(const float* __restrict__ O, const float* __restrict__ m,
                                                        const float* __restrict__ l, const int32_t* meta, float* out,
                                                        int32_t* lens, int B, int d, int dh) {
  pdl_wait_primary();
  pdl_launch_dependents();
  const int CT = d / kABN, b = blockIdx.x / CT, ct = blockIdx.x - b * CT;
  const int c = threadIdx.x, j = c / dh;
  const int lo = __ldcg(meta + 1 + b), hi = __ldcg(meta + 2 + b);
  float M = -INFINITY;
  for (int rt = lo; rt < hi; ++rt) M = fmaxf(M, __ldcg(m + (static_cast<size_t>(rt) * CT + ct) * 4 + j));
  float S = 0.f, acc = 0.f;
  for (int rt = lo; rt < hi; ++rt) {
    const size_t tau = static_cast<size_t>(rt) * CT + ct;
    const float w = exp2f(__ldcg(m + tau * 4 + j) - M);
    S = fmaf(w, __ldcg(l + tau * 4 + j), S);
    acc = fmaf(w, __ldcg(O + tau * kABN + c), acc);
  }
  out[static_cast<size_t>(b) * d + ct * kABN + c] = S > 0.f ? acc / S : 0.f;
  if (ct == 0 && c == 0 && (__ldcg(meta + 2 + B + b) & kSeqAppend)) lens[b] += 1;
}

}  // namespace

bool decode_a_tc_supported(int dtype, int B, int d, int H) {
  if (dtype != SLIM_BF16 || H <= 0 || d % H || d % kABN) return false;
  const int dh = d / H;
  if (dh != 64 && dh != 128) return false;
  return atc_smem_layout(B).total <= static_cast<uint32_t>(max_smem_optin());
}

// Partial slots (tiles) the workspace must hold: every sequence's row tiles times the column groups.
size_t decode_a_tc_slots(int B, int d, int64_t cap) {
  return static_cast<size_t>((static_cast<int64_t>(B) * (cap + 1) + kABM - 1) / kABM + B) * (d / kABN);
}

cudaError_t launch_decode_a_tc(const DecodeArgs& a, const SplitWorkspace& ws, cudaStream_t st, int* launches);

cudaError_t launch_decode_a_tc(const DecodeArgs& a, const SplitWorkspace& ws, cudaStream_t st, int* launches) {
  // K cache as {d columns, B·cap rows}, box 64 x 128, 128-byte swizzle (the A operand)
  CUtensorMap kmap, wmap;
  if (!encode_tmap_2d_bf16(&kmap, a.kcache, static_cast<uint64_t>(a.d), static_cast<uint64_t>(a.B) * a.cap,
                           static_cast<uint64_t>(a.d) * 2u, kABK, kABM, true))
    return cudaErrorInvalidValue;
  // W_KV as {64 columns, d rows, d/64 column blocks}, box 64 x 64 x 4 (the MN-major B operand)
  if (!encode_tmap_3d_bf16(&wmap, a.w_kv, 64, static_cast<uint64_t>(a.d), static_cast<uint64_t>(a.d / 64),
                           static_cast<uint64_t>(a.d) * 2u, 128u, 64, kABK, kABN / 64))
    return cudaErrorInvalidValue;
  DecodeATCParams prm;
  prm.q = a.q;
  prm.lens = a.lens;
  prm.status = a.status;
  prm.ws_O = ws.U;
  prm.ws_m = ws.m;
  prm.ws_l = ws.l;
  prm.ws_meta = ws.meta;
  prm.B = a.B;
  prm.d = a.d;
  prm.H = a.H;
  prm.cap = a.cap;
  prm.append = a.k_new != nullptr ? 1 : 0;
  prm.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(a.d / a.H));
  const uint32_t smem = atc_smem_layout(a.B).total;
  cudaError_t e = cudaFuncSetAttribute(decode_a_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(num_sms()), 1, 1);
  cfg.blockDim = dim3(kAThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, decode_a_tc_kernel, kmap, wmap, prm);
  if (e != cudaSuccess) return e;
  if (launches) ++*launches;
  cudaLaunchConfig_t cfg2 = {};
  cfg2.gridDim = dim3(static_cast<unsigned>(a.B * (a.d / kABN)), 1, 1);
  cfg2.blockDim = dim3(kABN, 1, 1);
  cfg2.stream = st;
  cfg2.attrs = attr;
  cfg2.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg2, merge_a_kernel, static_cast<const float*>(ws.U), static_cast<const float*>(ws.m),
                         static_cast<const float*>(ws.l), static_cast<const int32_t*>(ws.meta), a.out, a.lens, a.B,
                         a.d, a.d / a.H);
  if (e != cudaSuccess) return e;
  if (launches) ++*launches;
  return cudaSuccess;
}

}  // namespace slim
