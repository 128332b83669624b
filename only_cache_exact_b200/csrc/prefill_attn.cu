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
// This kernel is the attention part, flash-attention style on warp-level
// tensor-core MMAs (mma.sync m16n8k16, bf16 in, fp32 accumulation): a CTA owns
// 64 queries of one head of one sequence (16 per warp), streams 64-row tiles
// of K and V (TMA, 128-byte swizzle, 3-stage ring, bounded waits), computes
// S = Q·K^T, keeps a running max and sum per query row in registers, and adds
// P·V into register accumulators; the score accumulators are reused as the A
// operand of P·V without leaving registers.
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace slim {

namespace {

constexpr int kPQ = 64;       // queries per CTA
constexpr int kPK = 64;       // keys per tile
constexpr int kPStages = 3;
constexpr int kPThreads = 128;

struct PrefillAttnParams {
  float* out;           // [B][n][d]
  const int32_t* lens;  // the prompt's rows are the last n cached rows of every sequence
  int32_t* status;
  int B, n, d, H;
  int64_t cap;
  float scale_log2;
};

__host__ __device__ inline uint32_t pa_tile_bytes(int dhb) { return kPK * 128u * dhb; }
__host__ __device__ inline uint32_t pa_smem_bytes(int dhb) {
  return pa_tile_bytes(dhb) /*Q*/ + kPStages * 2u * pa_tile_bytes(dhb) /*K, V*/ + (1u + kPStages) * 8u + 1024u;
}

// byte offset of (row r, column c) in a tile of 64 rows x 64·DHB columns: [c / 64 boxes][64 rows][128 B], swizzled
__device__ __forceinline__ uint32_t pa_off(int r, int c) {
  return static_cast<uint32_t>((c >> 6) * (kPK * 128) + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}

template <int DHB>
__global__ void __launch_bounds__(kPThreads)
    prefill_attn_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                        const __grid_constant__ CUtensorMap vmap, const PrefillAttnParams p) {
  extern __shared__ uint8_t pa_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(pa_raw) + 1023) & ~uintptr_t(1023));
  constexpr int DH = 64 * DHB;
  constexpr int NTO = DH / 8;  // 8-column tiles of the output
  const uint32_t TB = pa_tile_bytes(DHB);
  uint8_t* qs = sm;
  uint8_t* kvs = sm + TB;  // [stage][K tile, V tile]
  uint64_t* qbar = reinterpret_cast<uint64_t*>(sm + TB + kPStages * 2u * TB);
  uint64_t* full = qbar + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, tq = lane & 3;

  // heaviest query tiles (the last ones) first
  const int nqt = (p.n + kPQ - 1) / kPQ;
  const int bh = blockIdx.x % (p.B * p.H);
  const int qt = nqt - 1 - blockIdx.x / (p.B * p.H);
  const int b = bh / p.H, h = bh - b * p.H;
  const int q0 = qt * kPQ;
  const int L = __ldg(p.lens + b);
  const int pos0 = L - p.n;  // position of query 0
  if (pos0 < 0 || static_cast<int64_t>(L) > p.cap) {
    if (threadIdx.x == 0 && h == 0 && qt == 0) atomicOr(p.status, SLIM_DEV_BADLEN);
    return;
  }
  const int last_key = pos0 + min(q0 + kPQ, p.n) - 1;  // largest position any query here attends
  const int nkt = last_key / kPK + 1;

  int issued = 0;
  auto issue = [&](int j) {  // K and V rows 64 j .. of this head into stage j % kPStages
    uint8_t* dst = kvs + (j % kPStages) * 2u * TB;
    uint64_t* bar = &full[j % kPStages];
    mbar_arrive_expect_tx(bar, 2u * TB);
    const int y = static_cast<int>(static_cast<int64_t>(b) * p.cap + j * kPK);
#pragma unroll
    for (int i = 0; i < DHB; ++i) {
      tma_load_2d(dst + i * (kPK * 128), &kmap, h * DH + 64 * i, y, bar, l2_policy_evict_last());
      tma_load_2d(dst + TB + i * (kPK * 128), &vmap, h * DH + 64 * i, y, bar, l2_policy_evict_last());
    }
    ++issued;
  };
  if (threadIdx.x == 0) {
    mbar_init(qbar, 1);
    for (int s = 0; s < kPStages; ++s) mbar_init(&full[s], 1);
    fence_barrier_init();
    tma_prefetch_desc(&qmap);
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&vmap);
    mbar_arrive_expect_tx(qbar, TB);
#pragma unroll
    for (int i = 0; i < DHB; ++i)
      tma_load_2d(qs + i * (kPK * 128), &qmap, h * DH + 64 * i, b * p.n + q0, qbar, l2_policy_evict_first());
    for (int j = 0; j < min(kPStages, nkt); ++j) issue(j);
  }
  __syncthreads();

  float o[NTO][4];
#pragma unroll
  for (int i = 0; i < NTO; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[i][e] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};  // rows g and g + 8 of the warp
  const int qr0 = q0 + warp * 16 + g;                           // query index of row g
  const int pr[2] = {pos0 + qr0, pos0 + qr0 + 8};              // their positions
  const uint32_t qbase = smem_u32(qs);
  bool ok = mbar_wait(qbar, 0u, p.status);
  int done = 0;
  for (int j = 0; j < nkt; ++j) {
    const int s = j % kPStages;
    const bool got = ok && mbar_wait(&full[s], static_cast<uint32_t>(j / kPStages) & 1u, p.status);
    ok = __syncthreads_and(got);
    if (!ok) break;
    const uint32_t kb = smem_u32(kvs + s * 2u * TB), vb = kb + TB;
    if ((j + 1) * kPK > L) {
      // rows at or past the sequence's length hold no key or value (the V buffer is scratch there):
      // zero them so that a masked score's p = 0 never meets a non-finite value
      uint8_t* kt = kvs + s * 2u * TB;
      const int r0 = L - j * kPK;
      for (int i = threadIdx.x; i < (kPK - r0) * 8 * DHB; i += kPThreads) {
        const int r = r0 + i / (8 * DHB), ch = i % (8 * DHB);
        const uint32_t off = pa_off(r, ch * 8);
        *reinterpret_cast<uint4*>(kt + off) = make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(kt + TB + off) = make_uint4(0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();  // these writes come before the stage's next TMA fill
      __syncthreads();
    }
    // S = Q·K^T for the warp's 16 queries x 64 keys
    float sc[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[nt][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < DH / 16; ++ks) {
      uint32_t a[4];
      {
        const int r = warp * 16 + (lane & 15), c = ks * 16 + (lane >> 4) * 8;
        ldsm_x4(qbase + pa_off(r, c), a[0], a[1], a[2], a[3]);
      }
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        uint32_t b0, b1;
        const int r = nt * 8 + (lane & 7), c = ks * 16 + ((lane >> 3) & 1) * 8;
        ldsm_x2(kb + pa_off(r, c), b0, b1);
        mma_16816_bf16(sc[nt], a, b0, b1);
      }
    }
    // causal mask, running max and sum (log2 domain), P in place
    const int k0 = j * kPK;
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = k0 + nt * 8 + 2 * tq + (e & 1);
        const int rr = e >> 1;
        const float v = key <= pr[rr] ? sc[nt][e] * p.scale_log2 : -INFINITY;
        sc[nt][e] = v;
        mx[rr] = fmaxf(mx[rr], v);
      }
    float alpha[2];
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      mx[rr] = fmaxf(mx[rr], __shfl_xor_sync(0xffffffffu, mx[rr], 1));
      mx[rr] = fmaxf(mx[rr], __shfl_xor_sync(0xffffffffu, mx[rr], 2));
      const float mn = fmaxf(mrow[rr], mx[rr]);
      alpha[rr] = mn == -INFINITY ? 1.f : exp2f(mrow[rr] - mn);
      mrow[rr] = mn;
      lrow[rr] *= alpha[rr];
    }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int rr = e >> 1;
        const float pv = mrow[rr] == -INFINITY ? 0.f : exp2f(sc[nt][e] - mrow[rr]);
        sc[nt][e] = pv;
        lrow[rr] += pv;
      }
#pragma unroll
    for (int i = 0; i < NTO; ++i) {
      o[i][0] *= alpha[0];
      o[i][1] *= alpha[0];
      o[i][2] *= alpha[1];
      o[i][3] *= alpha[1];
    }
    // O += P·V: P (16 x 64) from the score accumulators, V (64 keys x d_h) by transposed loads
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {  // 16 keys at a time
      uint32_t a[4];
      a[0] = pack_bf16x2(sc[2 * kk][0], sc[2 * kk][1]);
      a[1] = pack_bf16x2(sc[2 * kk][2], sc[2 * kk][3]);
      a[2] = pack_bf16x2(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
      a[3] = pack_bf16x2(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
#pragma unroll
      for (int nt = 0; nt < NTO; ++nt) {
        uint32_t b0, b1;
        const int r = kk * 16 + (lane & 15), c = nt * 8;
        ldmatrix_x2_trans(vb + pa_off(r, c), b0, b1);
        mma_16816_bf16(o[nt], a, b0, b1);
      }
    }
    done = j + 1;
    __syncthreads();  // every warp is done with the stage
    if (threadIdx.x == 0 && j + kPStages < nkt) issue(j + kPStages);
  }
  if (!ok && threadIdx.x == 0) {
    // copies still landing in this CTA's shared memory must complete before it exits
    mbar_wait(qbar, 0u, p.status);
    for (int j = done; j < issued; ++j)
      mbar_wait(&full[j % kPStages], static_cast<uint32_t>(j / kPStages) & 1u, p.status);
  }
  // o / l, rows of the warp's queries that exist
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    lrow[rr] += __shfl_xor_sync(0xffffffffu, lrow[rr], 1);
    lrow[rr] += __shfl_xor_sync(0xffffffffu, lrow[rr], 2);
  }
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const int qi = qr0 + 8 * rr;
    if (qi >= p.n) continue;
    const float inv = (ok && lrow[rr] > 0.f) ? 1.f / lrow[rr] : 0.f;
    float* dst = p.out + (static_cast<size_t>(b) * p.n + qi) * p.d + h * DH;
#pragma unroll
    for (int nt = 0; nt < NTO; ++nt)
      *reinterpret_cast<float2*>(dst + nt * 8 + 2 * tq) = make_float2(o[nt][2 * rr] * inv, o[nt][2 * rr + 1] * inv);
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
  const unsigned grid = static_cast<unsigned>(B * H * ((n + kPQ - 1) / kPQ));
  kern<<<grid, kPThreads, smem, st>>>(qmap, kmap, vmap, prm);
  e = cudaGetLastError();
  if (e == cudaSuccess && launches) ++*launches;
  return e;
}

}  // namespace slim
