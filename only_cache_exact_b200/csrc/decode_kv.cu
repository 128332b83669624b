// Standard multi-head attention decode over explicit K and V caches: the
// comparison baseline for the Slim attention step (the Slim article and the
// paper's abstract claim up to 2x faster token generation when the step is
// memory-bandwidth-bound, because only K is read). It computes, for each
// sequence b and head h,
//     o[b, h-cols] = softmax(q_h · K_h^T / sqrt(d_h)) · V_h
// over the cached rows plus this step's appended k and v: the plain MHA step
// of the article's section "K-Cache is All You Need" before the rewrite.
//
// Heads are independent, so the work splits over head groups of 256 columns
// (4 heads at d_h = 64, 2 at d_h = 128) as well as over rows: each (sequence,
// head group) is one work sequence of the contiguous-share split
// (split_plan.cuh), and a CTA streams its segments' K and V tiles (32 rows x
// 256 columns each, TMA, 128-byte swizzle) once. Per CTA:
//   warp 0       TMA producer (K and V tiles of a stage complete on one barrier);
//   warps 1..4   scores and online softmax: warp 1 + j owns head j of the group,
//                lane t row t of the tile (q_h·K_t on the CUDA cores, exact
//                rescale per tile); they also write this step's k and v into
//                the tile and the caches (the append);
//   warps 5..12  P·V: thread c owns column c of the group:
//                o_c = alpha o_c + Σ_t p_t V_tc.
// The arithmetic is 4 flops per pair of K and V elements, far below the CUDA
// cores' rate per HBM byte: the kernel is bound by HBM like the K-only step,
// with twice the cache bytes.
#include <cuda_bf16.h>

#include "split_plan.cuh"

namespace slim {

constexpr int kKVCols = 256;  // columns of a head group
constexpr int kKVRows = 32;   // rows of a tile
constexpr int kKVStages = 4;
constexpr int kKVScoreWarps = 4;
constexpr int kKVPVWarps = 8;
constexpr int kKVThreads = (1 + kKVScoreWarps + kKVPVWarps) * 32;
constexpr uint32_t kKVTileBytes = kKVRows * kKVCols * 2u;  // one of K or V

struct DecodeKVParams {
  const float* q;
  const __nv_bfloat16* k_new;
  const __nv_bfloat16* v_new;
  __nv_bfloat16* kcache;
  __nv_bfloat16* vcache;
  const int32_t* lens;
  int32_t* status;
  float* ws_O;  // [slots][256] unnormalised p·V of the group's columns
  float* ws_m;  // [slots][4] running max (log2 domain) per head of the group
  float* ws_l;  // [slots][4]
  int32_t* ws_meta;
  int B, d, H, HG;  // HG head groups per sequence
  int64_t cap;
  int append;
  int n_groups;
  int min_rows;
  float scale_log2;
};

struct KVSmem {
  uint32_t kv, p, alpha, q, bars, plan, total;
};
__host__ __device__ inline KVSmem kv_smem_layout(int Bw) {
  KVSmem s;
  uint32_t o = 0;
  s.kv = o;  // [stages][K tile, V tile], each [2 slabs][4 column blocks][16 rows][128 bytes]
  o += kKVStages * 2u * kKVTileBytes;
  s.p = o;  // [stages][4 heads][32 rows] fp32
  o += kKVStages * 4u * kKVRows * 4u;
  s.alpha = o;  // [stages][4 heads]
  o += kKVStages * 4u * 4u;
  s.q = o;  // [256] fp32, this segment's q columns
  o += kKVCols * 4u;
  s.bars = o;  // full, pready, empty per stage
  o += 3u * kKVStages * 8u;
  s.plan = o;  // s_nb, s_q, s_soff [Bw + 1] each, s_plan [2]
  o += (3u * static_cast<uint32_t>(Bw + 1) + 2u) * 4u;
  s.total = o + 1024u;
  return s;
}

// byte offset of element (row t, column c) in a tile: [slab t/16][block c/64][row t%16][128 B], swizzled
__device__ __forceinline__ uint32_t kv_off(int t, int c) {
  return static_cast<uint32_t>((t >> 4) * 8192 + (c >> 6) * 2048 + (t & 15) * 128 +
                               ((((c & 63) >> 3) ^ (t & 7)) << 4) + (c & 7) * 2);
}

template <int DHB>
__global__ void __launch_bounds__(kKVThreads, 1)
    decode_kv_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                     const DecodeKVParams p) {
  extern __shared__ uint8_t kvsm_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(kvsm_raw) + 1023) & ~uintptr_t(1023));
  constexpr int DH = 64 * DHB;
  constexpr int HPG = kKVCols / DH;  // heads of a group
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Bw = p.B * p.HG;
  const KVSmem L = kv_smem_layout(Bw);
  uint8_t* kv = sm + L.kv;
  float* p_s = reinterpret_cast<float*>(sm + L.p);
  float* alpha_s = reinterpret_cast<float*>(sm + L.alpha);
  float* q_s = reinterpret_cast<float*>(sm + L.q);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L.bars);
  uint64_t* pready = full + kKVStages;
  uint64_t* empty = pready + kKVStages;
  int* s_nb = reinterpret_cast<int*>(sm + L.plan);
  unsigned* s_q = reinterpret_cast<unsigned*>(s_nb + (Bw + 1));
  unsigned* s_soff = s_q + (Bw + 1);
  unsigned* s_plan = s_soff + (Bw + 1);

  if (threadIdx.x == 0) {
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&vmap);
    for (int s = 0; s < kKVStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&pready[s], kKVScoreWarps);
      mbar_init(&empty[s], kKVPVWarps);
    }
    fence_barrier_init();
  }
  pdl_wait_primary();
  pdl_launch_dependents();
  if (warp == 0)
    plan_lean(p.lens, Bw, p.HG, p.cap, p.append, p.n_groups, p.min_rows, s_nb, s_q, s_soff, s_plan, p.ws_meta,
              p.status, blockIdx.x == 0);
  __syncthreads();
  LeanCursor cur;
  cur.init(blockIdx.x, Bw, s_q, s_plan);
  SplitItem it;
  auto tiles_of = [](const SplitItem& x) { return (x.row1 - x.row0 + kKVRows - 1) / kKVRows; };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_first();
      int g = 0;
      bool ok = true;
      while (ok && cur.next(it, s_nb, s_q, s_soff)) {
        const int b = it.b / p.HG, hg = it.b - b * p.HG;
        const int nt = tiles_of(it);
        for (int t = 0; t < nt; ++t, ++g) {
          const int s = g % kKVStages;
          const uint32_t ph = static_cast<uint32_t>(g / kKVStages) & 1u;
          if (g >= kKVStages && !mbar_wait(&empty[s], ph ^ 1u, p.status)) {
            ok = false;
            break;
          }
          const int r_lo = it.row0 + t * kKVRows;
          const int nbox = (min(kKVRows, it.row1 - r_lo) + 15) / 16;
          mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(nbox) * 2u * (kKVTileBytes / 2u));
          const int y0 = static_cast<int>(static_cast<int64_t>(b) * p.cap + r_lo);
          uint8_t* dk = kv + s * 2u * kKVTileBytes;
          for (int rb = 0; rb < nbox; ++rb) {
            tma_load_3d(dk + rb * 8192, &kmap, 0, y0 + rb * 16, hg * 4, &full[s], pol);
            tma_load_3d(dk + kKVTileBytes + rb * 8192, &vmap, 0, y0 + rb * 16, hg * 4, &full[s], pol);
          }
        }
      }
      for (int t = max(0, g - kKVStages); t < g; ++t)  // drain: every issued copy lands before exit
        mbar_wait(&full[t % kKVStages], static_cast<uint32_t>(t / kKVStages) & 1u, p.status);
    }
  } else if (warp <= kKVScoreWarps) {
    // ------------------------------------------------------------ scores, softmax, append
    const int j = warp - 1;  // head of the group; lane = row of the tile
    const bool has_head = j < HPG;
    int g = 0;
    bool ok = true;
    while (ok && cur.next(it, s_nb, s_q, s_soff)) {
      const int b = it.b / p.HG, hg = it.b - b * p.HG;
      const int nt = tiles_of(it);
      const int nb_old = it.nb - p.append;
      const int col0 = hg * kKVCols;
      // q of the group's columns (warps 1..4 load 64 each)
      reinterpret_cast<float2*>(q_s)[j * 32 + lane] =
          __ldg(reinterpret_cast<const float2*>(p.q + static_cast<size_t>(b) * p.d + col0) + j * 32 + lane);
      named_barrier_sync(1, kKVScoreWarps * 32);
      float mref = -INFINITY, lsum = 0.f;
      for (int t = 0; t < nt; ++t, ++g) {
        const int s = g % kKVStages;
        const uint32_t ph = static_cast<uint32_t>(g / kKVStages) & 1u;
        // one decision for the four score warps, so their named barriers stay aligned
        if (!named_barrier_and(1, kKVScoreWarps * 32, __all_sync(0xffffffffu, mbar_wait(&full[s], ph, p.status)))) {
          ok = false;
          break;
        }
        uint8_t* kt = kv + s * 2u * kKVTileBytes;
        uint8_t* vt = kt + kKVTileBytes;
        const int r_lo = it.row0 + t * kKVRows;
        const int nvalid = min(kKVRows, it.row1 - r_lo);
        const int nloaded = (nvalid + 15) & ~15;
        if (r_lo + nloaded > nb_old) {
          // rows at or after nb_old hold no cached key: this step's k and v go to row nb_old (tile
          // and caches), the rest become zero. The four warps split the 256 columns.
          const int fr0 = max(nb_old - r_lo, 0);
          for (int i = lane; i < (nloaded - fr0) * 8; i += 32) {
            const int rw = fr0 + (i >> 3), c = j * 64 + (i & 7) * 8;
            uint4 kvv = make_uint4(0u, 0u, 0u, 0u), vvv = make_uint4(0u, 0u, 0u, 0u);
            if (p.append && r_lo + rw == nb_old) {
              const size_t src = static_cast<size_t>(b) * p.d + col0 + c;
              const size_t dst = (static_cast<size_t>(b) * p.cap + nb_old) * p.d + col0 + c;
              kvv = __ldg(reinterpret_cast<const uint4*>(p.k_new + src));
              vvv = __ldg(reinterpret_cast<const uint4*>(p.v_new + src));
              *reinterpret_cast<uint4*>(p.kcache + dst) = kvv;
              *reinterpret_cast<uint4*>(p.vcache + dst) = vvv;
            }
            *reinterpret_cast<uint4*>(kt + kv_off(rw, c)) = kvv;
            *reinterpret_cast<uint4*>(vt + kv_off(rw, c)) = vvv;
          }
          fence_proxy_async_smem();  // these writes come before the stage's next TMA fill
          named_barrier_sync(1, kKVScoreWarps * 32);  // every column fixed before the scores read K
        }
        float sc = -INFINITY;
        if (has_head && lane < nvalid) {
          float a0 = 0.f, a1 = 0.f;
#pragma unroll
          for (int c8 = 0; c8 < DH / 8; ++c8) {
            const int c = j * DH + c8 * 8;
            const uint4 kw = *reinterpret_cast<const uint4*>(kt + kv_off(lane, c));
            const float4 qa = *reinterpret_cast<const float4*>(q_s + c);
            const float4 qb = *reinterpret_cast<const float4*>(q_s + c + 4);
            a0 = fmaf(bf16lo(kw.x), qa.x, a0);
            a1 = fmaf(bf16hi(kw.x), qa.y, a1);
            a0 = fmaf(bf16lo(kw.y), qa.z, a0);
            a1 = fmaf(bf16hi(kw.y), qa.w, a1);
            a0 = fmaf(bf16lo(kw.z), qb.x, a0);
            a1 = fmaf(bf16hi(kw.z), qb.y, a1);
            a0 = fmaf(bf16lo(kw.w), qb.z, a0);
            a1 = fmaf(bf16hi(kw.w), qb.w, a1);
          }
          sc = (a0 + a1) * p.scale_log2;
        }
        const float mx = warp_max(sc);
        float alpha = 1.f, pv = 0.f;
        if (has_head) {
          const float mnew = fmaxf(mref, mx);
          alpha = mref == -INFINITY ? 1.f : exp2f(mref - mnew);
          mref = mnew;
          pv = lane < nvalid ? exp2f(sc - mnew) : 0.f;
          lsum = fmaf(lsum, alpha, pv);
        }
        p_s[(s * 4 + j) * kKVRows + lane] = pv;
        if (lane == 0) alpha_s[s * 4 + j] = alpha;
        __syncwarp();
        if (lane == 0) mbar_arrive(&pready[s]);
      }
      if (!ok) break;
      const float tot = warp_sum(lsum);
      if (has_head && lane == 0) {
        p.ws_m[static_cast<size_t>(it.slot) * 4 + j] = mref;
        p.ws_l[static_cast<size_t>(it.slot) * 4 + j] = tot;
      }
      named_barrier_sync(1, kKVScoreWarps * 32);  // q_s is reloaded by the next segment
    }
  } else {
    // ------------------------------------------------------------ P·V
    const int c = (warp - 1 - kKVScoreWarps) * 32 + lane;  // column of the group
    const int j = c / DH;
    int g = 0;
    bool ok = true;
    while (ok && cur.next(it, s_nb, s_q, s_soff)) {
      const int nt = tiles_of(it);
      float o = 0.f;
      for (int t = 0; t < nt; ++t, ++g) {
        const int nvalid = min(kKVRows, it.row1 - it.row0 - t * kKVRows);  // rows past it were not loaded
        const int s = g % kKVStages;
        const uint32_t ph = static_cast<uint32_t>(g / kKVStages) & 1u;
        if (!__all_sync(0xffffffffu, mbar_wait(&pready[s], ph, p.status))) {
          ok = false;
          break;
        }
        const uint8_t* vt = kv + s * 2u * kKVTileBytes + kKVTileBytes;
        const float* pr = p_s + (s * 4 + j) * kKVRows;
        float a = o * alpha_s[s * 4 + j];
#pragma unroll 8
        for (int r = 0; r < nvalid; ++r) {
          const uint16_t v = *reinterpret_cast<const uint16_t*>(vt + kv_off(r, c));
          a = fmaf(pr[r], __uint_as_float(static_cast<uint32_t>(v) << 16), a);
        }
        o = a;
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
      if (!ok) break;
      p.ws_O[static_cast<size_t>(it.slot) * kKVCols + c] = o;
    }
  }
  __syncwarp();
  __syncthreads();
}

// Merge of the head groups' partials: out[b, hg·256 + c] = Σ_s 2^(m_s - M) O_s[c] / Σ_s 2^(m_s - M) l_s
// over the slots s of work sequence (b, hg); one CTA per work sequence, one thread per column.
// The lengths advance here (after every split CTA has read them).
__global__ void __launch_bounds__(kKVCols) merge_kv_kernel(const float* __restrict__ O, const float* __restrict__ m,
                                                            const float* __restrict__ l, const int32_t* meta,
                                                            float* out, int32_t* lens, int B, int d, int HG, int dh) {
  pdl_wait_primary();
  pdl_launch_dependents();
  const int vb = blockIdx.x, b = vb / HG, hg = vb - b * HG;
  const int c = threadIdx.x, j = c / dh;
  const int Bw = B * HG;
  const int lo = __ldcg(meta + 1 + vb), hi = __ldcg(meta + 2 + vb);
  float M = -INFINITY;
  for (int s = lo; s < hi; ++s) M = fmaxf(M, __ldcg(m + static_cast<size_t>(s) * 4 + j));
  float S = 0.f, acc = 0.f;
  for (int s = lo; s < hi; ++s) {
    const float w = exp2f(__ldcg(m + static_cast<size_t>(s) * 4 + j) - M);
    S = fmaf(w, __ldcg(l + static_cast<size_t>(s) * 4 + j), S);
    acc = fmaf(w, __ldcg(O + static_cast<size_t>(s) * kKVCols + c), acc);
  }
  out[static_cast<size_t>(b) * d + hg * kKVCols + c] = S > 0.f ? acc / S : 0.f;
  if (hg == 0 && c == 0 && (__ldcg(meta + 2 + Bw + vb) & kSeqAppend)) lens[b] += 1;
}

// ---------------------------------------------------------------------------- host
bool decode_kv_supported(int B, int d, int H, int64_t cap) {
  if (H <= 0 || d % H || d % kKVCols) return false;
  const int dh = d / H;
  if (dh != 64 && dh != 128) return false;
  if (static_cast<int64_t>(B) * (d / kKVCols) * cap > (int64_t(1) << 31) - 1) return false;
  return kv_smem_layout(B * (d / kKVCols)).total <= static_cast<uint32_t>(max_smem_optin());
}

size_t kv_ws_slots(int B, int d) { return static_cast<size_t>(num_sms()) + static_cast<size_t>(B) * (d / kKVCols); }

cudaError_t launch_decode_kv(const float* q, const void* k_new, const void* v_new, void* kcache, void* vcache,
                             int32_t* lens, int B, int d, int H, int64_t cap, float* out, float* wsO, float* wsm,
                             float* wsl, int32_t* meta, int32_t* status, cudaStream_t st, int* launches) {
  const int HG = d / kKVCols, dh = d / H;
  CUtensorMap kmap, vmap;
  if (!encode_tmap_kslab(&kmap, kcache, static_cast<uint64_t>(B) * cap, d, 4) ||
      !encode_tmap_kslab(&vmap, vcache, static_cast<uint64_t>(B) * cap, d, 4))
    return cudaErrorInvalidValue;
  DecodeKVParams prm;
  prm.q = q;
  prm.k_new = static_cast<const __nv_bfloat16*>(k_new);
  prm.v_new = static_cast<const __nv_bfloat16*>(v_new);
  prm.kcache = static_cast<__nv_bfloat16*>(kcache);
  prm.vcache = static_cast<__nv_bfloat16*>(vcache);
  prm.lens = lens;
  prm.status = status;
  prm.ws_O = wsO;
  prm.ws_m = wsm;
  prm.ws_l = wsl;
  prm.ws_meta = meta;
  prm.B = B;
  prm.d = d;
  prm.H = H;
  prm.HG = HG;
  prm.cap = cap;
  prm.append = k_new != nullptr ? 1 : 0;
  prm.n_groups = num_sms();
  prm.min_rows = 64;
  prm.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(dh));
  const uint32_t smem = kv_smem_layout(B * HG).total;
  auto kern = dh == 64 ? decode_kv_kernel<1> : decode_kv_kernel<2>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(prm.n_groups), 1, 1);
  cfg.blockDim = dim3(kKVThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, kmap, vmap, prm);
  if (e != cudaSuccess) return e;
  if (launches) ++*launches;
  cudaLaunchConfig_t cfg2 = {};
  cfg2.gridDim = dim3(static_cast<unsigned>(B * HG), 1, 1);
  cfg2.blockDim = dim3(kKVCols, 1, 1);
  cfg2.stream = st;
  cfg2.attrs = attr;
  cfg2.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg2, merge_kv_kernel, static_cast<const float*>(wsO), static_cast<const float*>(wsm),
                         static_cast<const float*>(wsl), static_cast<const int32_t*>(meta), out, lens, B, d, HG, dh);
  if (e != cudaSuccess) return e;
  if (launches) ++*launches;
  return cudaSuccess;
}

}  // namespace slim
