// Prompt-phase attention output over the K-only cache (bf16, d_h = 64 or 128).
//
// Slim Attention article, section "K-Cache is All You Need", prompt phase: the
// queries and keys of all prompt tokens are formed in parallel and only K is
// cached; the values come from K through W_KV. In the prompt phase the first
// ordering of the generation phase is the cheap one: V = K·W_KV is computed
// once for the rows (a tcgen05 GEMM, gemm_tc.cu) and every one of the n
// queries reuses it, where contracting each query's softmax row with K first
// would cost 2·H·d per key and query. The output is causal attention:
//     o_i = softmax(q_i · K_{<=p_i}^T / sqrt(d_h)) · V_{<=p_i}
// per head, p_i the position of query i (its own key included).
//
// This kernel is the attention part, flash-attention style on tcgen05 tensor cores: a CTA owns two
// adjacent 128-query tiles of one head of one sequence and walks the 128-key tiles up to its last
// query's position; every K and V tile it loads serves both query tiles.
//   warp 0     TMA producer: the two Q tiles once, then K and V tiles (128 rows x d_h, 128-byte
//              swizzle) through separate K and V rings of 2 (d_h = 128) or 6 stages; a K stage is
//              released when the last S MMA that reads it completes, a V stage with the last P·V
//   warp 1     tcgen05.mma issuer, per query tile t: S_t = Q_t·K^T (M = 128 queries, N = 128 keys,
//              K = d_h) into the tile's 128-column TMEM S region; O_t += P_t·V (M = 128, N = d_h,
//              K = 128 keys) into the tile's O region, P_t read from tensor memory (the first 64
//              columns of the S region, bf16 pairs) and V in place from shared memory as the
//              MN-major operand. Issue order P_0(j)·V_j, S_0(j+1), P_1(j)·V_j, S_1(j+1): while one
//              tile's softmax runs, the tensor cores work through the other tile's MMAs.
//   warps 2-5  softmax of query tile 0, warps 6-9 of query tile 1, one query row per thread (TMEM
//              lane = row; warp w reads lanes 32 (w mod 4) ..): the tile's scores, the causal mask, a
//              running max kept lazily (O is rescaled in TMEM only when a row's max grows by more
//              than 2^8, so P <= 2^8 stays exact enough in bf16), P in bf16 over the S region in
//              tensor memory, the row sums in fp32 registers; at the end o = O / l to global memory.
// The tensor cores run one CTA's MMAs in issue order, so the S MMA that next writes a tile's S
// region (issued after the P·V MMA that reads the P stored there) never overwrites P before it is
// read.
// Key rows at or past a sequence's length are scratch in the V buffer: their rows of the last
// tile are zeroed in shared memory before the first P·V MMA that reads them (a masked score's
// p = 0 never meets a non-finite value).
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace slim {

namespace {

constexpr int kPQ = 128;  // queries per query tile (the MMA's M)
constexpr int kPK = 128;  // keys per key tile (the S MMA's N)
constexpr int kPT = 2;    // query tiles per CTA
constexpr int kPThreads = 64 + 128 * kPT;  // producer warp, MMA warp, a softmax warpgroup per query tile
constexpr uint32_t kPTmemPerTile = 256;    // S (and P over it) at columns 0..127, O at 128
constexpr float kPLazyLog2 = 8.f;

struct PrefillAttnParams {
  float* out;           // [B][n][d]
  const int32_t* lens;  // the prompt's rows are the last n cached rows of every sequence
  int32_t* status;
  int B, n, d, H;
  int64_t cap;
  float scale_log2;
};

__host__ __device__ inline int pa_stages(int dhb) { return dhb == 2 ? 2 : 6; }

// 2^x on the special-function unit (the PTX approximate base-2 exponential; subnormal results flush
// to zero, which for a softmax weight below 2^-126 is a zero weight).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__host__ __device__ inline uint32_t pa_q_bytes(int dhb) { return 128u * 128u * dhb; }   // 128 queries x d_h bf16
__host__ __device__ inline uint32_t pa_kv_bytes(int dhb) { return 128u * 128u * dhb; }  // 128 keys x d_h bf16
__host__ __device__ inline uint32_t pa_smem_bytes(int dhb) {
  // the Q tiles, the K and V rings, barriers, TMEM slot; slack for 1024-byte alignment
  return kPT * pa_q_bytes(dhb) + pa_stages(dhb) * 2u * pa_kv_bytes(dhb) + 512u + 1024u;
}

// 16 consecutive 32-bit TMEM columns of this thread's lane (32x32b shape, one lane per thread).
__device__ __forceinline__ void tmem_st16_u32(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

// D (TMEM) (+)= A · B with the bf16 A operand in tensor memory (K-major: row i in lane i, two
// elements per 32-bit column) and B from a shared-memory descriptor.
__device__ __forceinline__ void umma_f16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                                uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

template <int DHB>
__global__ void __launch_bounds__(kPThreads, 1)
    prefill_attn_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                        const __grid_constant__ CUtensorMap vmap, const PrefillAttnParams p) {
  extern __shared__ uint8_t pa_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(pa_raw) + 1023) & ~uintptr_t(1023));
  constexpr int DH = 64 * DHB;
  constexpr int NS = DHB == 2 ? 2 : 6;
  const uint32_t TQ = pa_q_bytes(DHB), T = pa_kv_bytes(DHB);
  uint8_t* qs = sm;                // [query tile][DHB boxes][128 rows][128 B]
  uint8_t* ks = sm + kPT * TQ;     // K ring: [stage][DHB boxes][128 rows][128 B]
  uint8_t* vs = ks + NS * T;       // V ring: [stage][DHB boxes][128 rows][128 B]
  uint64_t* bars = reinterpret_cast<uint64_t*>(vs + NS * T);
  uint64_t* qbar = bars;           // the Q tiles landed
  uint64_t* kfull = bars + 1;      // [NS] K of a key tile landed
  uint64_t* kempty = kfull + NS;   // [NS] the key tile's S MMAs completed
  uint64_t* vfull = kempty + NS;   // [NS] V of a key tile landed
  uint64_t* vempty = vfull + NS;   // [NS] the key tile's P·V MMAs completed
  uint64_t* sfull = vempty + NS;   // [query tile] S written
  uint64_t* pready = sfull + kPT;  // [query tile] S read, P written over it (and O rescaled) by the four warps
  uint64_t* pfree = pready + kPT;  // [query tile] the P·V MMA completed
  uint64_t* ofull = pfree + kPT;   // [query tile] the tile's last P·V MMA completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ofull + kPT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // heaviest query tiles (the last ones) first; the CTA's tiles are nqt - kPT (pair + 1) + t, a
  // negative index is an absent tile (an odd number of tiles)
  const int nqt = (p.n + kPQ - 1) / kPQ;
  const int bh = blockIdx.x % (p.B * p.H);
  const int pair = blockIdx.x / (p.B * p.H);
  const int b = bh / p.H, h = bh - b * p.H;
  const int L = __ldg(p.lens + b);
  const int pos0 = L - p.n;  // position of query 0
  if (pos0 < 0 || static_cast<int64_t>(L) > p.cap) {
    if (threadIdx.x == 0 && h == 0 && pair == 0) atomicOr(p.status, SLIM_DEV_BADLEN);
    return;
  }
  auto tile_q0 = [&](int t) { return (nqt - kPT * (pair + 1) + t) * kPQ; };
  // key tiles query tile t attends: up to its last query's position; 0 for an absent tile
  auto tile_keys = [&](int t) {
    const int q0 = tile_q0(t);
    return q0 < 0 ? 0 : (pos0 + min(q0 + kPQ, p.n) - 1) / kPK + 1;
  };
  const int nkt = tile_keys(kPT - 1);  // the last tile attends the most keys

  if (warp == 0 && lane == 0) {
    mbar_init(qbar, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&kfull[s], 1);
      mbar_init(&kempty[s], 1);
      mbar_init(&vfull[s], 1);
      mbar_init(&vempty[s], 1);
    }
    for (int t = 0; t < kPT; ++t) {
      mbar_init(&sfull[t], 1);
      mbar_init(&pready[t], 4);
      mbar_init(&pfree[t], 1);
      mbar_init(&ofull[t], 1);
    }
    fence_barrier_init();
  } else if (warp == 1) {
    tmem_alloc(tmem_slot, kPTmemPerTile * kPT);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&qmap);
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      uint32_t qbytes = 0;
#pragma unroll
      for (int t = 0; t < kPT; ++t)
        if (tile_keys(t) > 0) qbytes += TQ;
      mbar_arrive_expect_tx(qbar, qbytes);
#pragma unroll
      for (int t = 0; t < kPT; ++t) {
        if (tile_keys(t) == 0) continue;
#pragma unroll
        for (int i = 0; i < DHB; ++i)
          tma_load_2d(qs + t * TQ + i * 16384, &qmap, h * DH + 64 * i, b * p.n + tile_q0(t), qbar,
                      l2_policy_evict_first());
      }
      int nk_issued = 0, nv_issued = 0;
      for (int j = 0; j < nkt; ++j) {
        const int s = j % NS;
        const uint32_t ph = static_cast<uint32_t>((j / NS) & 1);
        const int y = static_cast<int>(static_cast<int64_t>(b) * p.cap + j * kPK);
        if (j >= NS && !mbar_wait(&kempty[s], ph ^ 1u, p.status)) break;
        mbar_arrive_expect_tx(&kfull[s], T);
#pragma unroll
        for (int i = 0; i < DHB; ++i)
          tma_load_2d(ks + s * T + i * 16384, &kmap, h * DH + 64 * i, y, &kfull[s], l2_policy_evict_last());
        ++nk_issued;
        if (j >= NS && !mbar_wait(&vempty[s], ph ^ 1u, p.status)) break;
        mbar_arrive_expect_tx(&vfull[s], T);
#pragma unroll
        for (int i = 0; i < DHB; ++i)
          tma_load_2d(vs + s * T + i * 16384, &vmap, h * DH + 64 * i, y, &vfull[s], l2_policy_evict_last());
        ++nv_issued;
      }
      // every issued copy lands before the CTA exits
      mbar_wait(qbar, 0u, p.status);
      for (int u = max(0, nk_issued - NS); u < nk_issued; ++u)
        mbar_wait(&kfull[u % NS], static_cast<uint32_t>(u / NS) & 1u, p.status);
      for (int u = max(0, nv_issued - NS); u < nv_issued; ++u)
        mbar_wait(&vfull[u % NS], static_cast<uint32_t>(u / NS) & 1u, p.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(kPQ, kPK, 0u, 0u);
      const uint32_t idesc_o = idesc_bf16_f32(kPQ, DH, 0u, 1u);
      const uint32_t qb = smem_u32(qs), kb0 = smem_u32(ks), vb0 = smem_u32(vs);
      int nk[kPT];
#pragma unroll
      for (int t = 0; t < kPT; ++t) nk[t] = tile_keys(t);
      bool ok = mbar_wait(qbar, 0u, p.status);
      // S_t(j) = Q_t·K_j^T into the tile's S region; the last tile's S MMA is the last reader of K_j
      auto issue_s = [&](int t, int j) {
        const int s = j % NS;
        if (!mbar_wait(&kfull[s], static_cast<uint32_t>(j / NS) & 1u, p.status)) return false;
        tc_fence_after();
        const uint32_t kb = kb0 + s * T, qtb = qb + t * TQ;
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          // Q and K both K-major (d_h contiguous): 64-column boxes 16 KB apart, 8-row groups 1024 B
          // apart, a 16-column step is 32 B into the swizzled row
          const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
          umma_f16(tmem + t * kPTmemPerTile, smem_desc(qtb + off, 16, 1024, kLayoutSW128),
                   smem_desc(kb + off, 16, 1024, kLayoutSW128), idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(&sfull[t]);
        if (t == kPT - 1) umma_commit(&kempty[s]);
        return true;
      };
      // O_t += P_t(j)·V_j; the last tile's P·V is the last reader of V_j
      auto issue_pv = [&](int t, int j) {
        const int s = j % NS;
        if (!mbar_wait(&pready[t], static_cast<uint32_t>(j) & 1u, p.status) ||
            !mbar_wait(&vfull[s], static_cast<uint32_t>(j / NS) & 1u, p.status))
          return false;
        tc_fence_after();
        const uint32_t vb = vb0 + s * T, pt = tmem + t * kPTmemPerTile;
#pragma unroll
        for (int kk = 0; kk < kPK / 16; ++kk) {
          // P in TMEM, 16 keys = 8 columns per step; V MN-major (d_h contiguous): 64-column blocks
          // 16 KB apart, 8-key groups 1024 B apart, 16 keys per step
          umma_f16_tmem_a(tmem + t * kPTmemPerTile + 128u, pt + static_cast<uint32_t>(kk * 8),
                          smem_desc(vb + kk * 2048u, 16384, 1024, kLayoutSW128), idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&pfree[t]);
        if (t == kPT - 1) umma_commit(&vempty[s]);
        return true;
      };
      bool committed[kPT];
#pragma unroll
      for (int t = 0; t < kPT; ++t) {
        committed[t] = false;
        if (ok && nk[t] > 0) ok = issue_s(t, 0);
      }
      for (int j = 0; ok && j < nkt; ++j) {
#pragma unroll
        for (int t = 0; t < kPT; ++t) {
          if (!ok || j >= nk[t]) continue;
          if (!issue_pv(t, j)) ok = false;
          if (ok && j == nk[t] - 1) {
            umma_commit(&ofull[t]);
            committed[t] = true;
          }
          // S_t(j+1) overwrites the P that the P·V above reads: issued after it
          if (ok && j + 1 < nk[t] && !issue_s(t, j + 1)) ok = false;
        }
      }
      // also after a failure: each output barrier covers every MMA issued
#pragma unroll
      for (int t = 0; t < kPT; ++t)
        if (!committed[t]) umma_commit(&ofull[t]);
#pragma unroll
      for (int t = 0; t < kPT; ++t) mbar_wait(&ofull[t], 0u, p.status);
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroup of query tile t
    const int t = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // query row of the tile = TMEM lane
    const uint32_t lrow = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t ts = tmem + t * kPTmemPerTile, tmem_o = ts + 128u;
    const int q0 = tile_q0(t), nkt_t = tile_keys(t);
    // the lowest tile that attends a key tile zeroes its rows past the length
    const int nkt_below = t > 0 ? tile_keys(t - 1) : 0;
    const int pos = pos0 + q0 + r;  // position of this row's query
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkt_t; ++j) {
      const int s = j % NS;
      if (!__all_sync(0xffffffffu, mbar_wait(&sfull[t], static_cast<uint32_t>(j) & 1u, p.status))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sc[kPK];
#pragma unroll
      for (int c = 0; c < kPK / 16; ++c)
        tmem_ld16(ts + lrow + static_cast<uint32_t>(16 * c), *reinterpret_cast<float(*)[16]>(sc + 16 * c));
      tmem_wait_ld();
      // keys past this query masked (only a tile that reaches past the query has any); the scale
      // is applied with the exponent below (max(s)·scale = max(s·scale) for scale > 0)
      const int k0 = j * kPK;
      if (k0 + kPK - 1 > pos) {
#pragma unroll
        for (int c = 0; c < kPK; ++c) sc[c] = (k0 + c <= pos) ? sc[c] : -INFINITY;
      }
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < kPK; ++c) mx[c & 3] = fmaxf(mx[c & 3], sc[c]);
      const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * p.scale_log2;
      float alpha = 1.f;
      if (j == 0 || m == -INFINITY) {
        m = mt;
      } else if (mt > m + kPLazyLog2) {
        alpha = ex2_approx(m - mt);
        m = mt;
        l *= alpha;
      }
      // P = 2^(s·scale - m) in bf16 over the S region, 32 keys (16 columns) at a time: keys 2c and
      // 2c + 1 in column c of the row's lane. The row sum adds the fp32 values before rounding (each
      // differs from the bf16 the MMA sees by at most 2^-9 relative, so l does too).
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
      const float nm = m == -INFINITY ? 0.f : -m;
#pragma unroll
      for (int q = 0; q < kPK / 32; ++q) {
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const float a = ex2_approx(fmaf(sc[32 * q + 2 * c], p.scale_log2, nm));
          const float bb = ex2_approx(fmaf(sc[32 * q + 2 * c + 1], p.scale_log2, nm));
          const __nv_bfloat162 hv = __floats2bfloat162_rn(a, bb);
          ls[c & 3] += a + bb;
          pk[c] = *reinterpret_cast<const uint32_t*>(&hv);
        }
        tmem_st16_u32(ts + lrow + static_cast<uint32_t>(16 * q), pk);
      }
      l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
      if (j >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
        // O is rescaled once the previous key tile's P·V has completed (after P, so that the scores
        // are no longer live)
        if (!__all_sync(0xffffffffu, mbar_wait(&pfree[t], static_cast<uint32_t>(j - 1) & 1u, p.status))) {
          tmem_wait_st();
          ok = false;
          break;
        }
        tc_fence_after();
        for (int c = 0; c < DH; c += 16) {
          float v[16];
          tmem_ld16(tmem_o + lrow + static_cast<uint32_t>(c), v);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] *= alpha;
          tmem_st16(tmem_o + lrow + static_cast<uint32_t>(c), v);
        }
      }
      tmem_wait_st();
      // key rows at or past the length in this key tile hold no value: zero them in V (thread r
      // takes key row r, once the tile's V has landed), unless a lower query tile attends this key
      // tile and zeroed them before its own P·V
      if (k0 + kPK > L && j >= nkt_below && k0 + r >= L) {
        if (mbar_wait(&vfull[s], static_cast<uint32_t>(j / NS) & 1u, p.status)) {
          uint8_t* vrow = vs + s * T + r * 128;
#pragma unroll
          for (int i = 0; i < DHB; ++i)
#pragma unroll
            for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(vrow + i * 16384 + c * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      fence_proxy_async_smem();  // zeroed V rows are read by the tensor cores
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&pready[t]);
    }
    // o = O / l
    if (nkt_t > 0) {
      const bool got = ok && __all_sync(0xffffffffu, mbar_wait(&ofull[t], 0u, p.status));
      tc_fence_after();
      const int qi = q0 + r;
      const float inv = (got && l > 0.f) ? 1.f / l : 0.f;
      float* dst = p.out + (static_cast<size_t>(b) * p.n + qi) * p.d + h * DH;
      for (int c = 0; c < DH; c += 16) {
        float v[16];
        tmem_ld16(tmem_o + lrow + static_cast<uint32_t>(c), v);
        tmem_wait_ld();
        if (qi < p.n) {
#pragma unroll
          for (int i = 0; i < 16; i += 4)
            *reinterpret_cast<float4*>(dst + c + i) = make_float4(v[i] * inv, v[i + 1] * inv, v[i + 2] * inv, v[i + 3] * inv);
        }
      }
    }
  }
  __syncwarp();  // lanes 1..31 of warps 0 and 1 skipped the lane-0 loops
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kPTmemPerTile * kPT);
  }
}

}  // namespace

bool prefill_attn_supported(int dtype, int d, int H) {
  if (dtype != SLIM_BF16 || H <= 0 || d % H) return false;
  const int dh = d / H;
  return (dh == 64 || dh == 128) && d % 256 == 0;
}

cudaError_t launch_prefill_attn(const void* Q, const void* kcache, const void* vbuf, const int32_t* lens, int B,
                                int n, int d, int H, int64_t cap, float* out, int32_t* status, cudaStream_t st,
                                int* launches) {
  const int dh = d / H, dhb = dh / 64;
  CUtensorMap qmap, kmap, vmap;
  if (!encode_tmap_2d_bf16(&qmap, Q, static_cast<uint64_t>(d), static_cast<uint64_t>(B) * n,
                           static_cast<uint64_t>(d) * 2u, 64, kPQ, true) ||
      !encode_tmap_2d_bf16(&kmap, kcache, static_cast<uint64_t>(d), static_cast<uint64_t>(B) * cap,
                           static_cast<uint64_t>(d) * 2u, 64, kPK, true) ||
      !encode_tmap_2d_bf16(&vmap, vbuf, static_cast<uint64_t>(d), static_cast<uint64_t>(B) * cap,
                           static_cast<uint64_t>(d) * 2u, 64, kPK, true))
    return cudaErrorInvalidValue;
  PrefillAttnParams prm;
  prm.out = out;
  prm.lens = lens;
  prm.status = status;
  prm.B = B;
  prm.n = n;
  prm.d = d;
  prm.H = H;
  prm.cap = cap;
  prm.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(dh));
  const uint32_t smem = pa_smem_bytes(dhb);
  auto kern = dhb == 1 ? prefill_attn_kernel<1> : prefill_attn_kernel<2>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int nqt = (n + kPQ - 1) / kPQ;
  const unsigned grid = static_cast<unsigned>(B * H * ((nqt + kPT - 1) / kPT));
  kern<<<grid, kPThreads, smem, st>>>(qmap, kmap, vmap, prm);
  e = cudaGetLastError();
  if (e == cudaSuccess && launches) ++*launches;
  return e;
}

}  // namespace slim
