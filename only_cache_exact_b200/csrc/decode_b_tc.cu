// Generation step, ordering (b), on tcgen05 tensor cores (bf16 K cache).
//
// Slim Attention article, section "K-Cache is All You Need", generation
// phase, second option: multiply the per-head softmax rows by K first (a full
// d-row per head) and only then by W_KV. Per work item (one row chunk of one
// sequence, see split_plan.cuh) this kernel streams the chunk's K rows once
// and produces the flash-decoding partial of every head h:
//     m_h = running max of the scaled scores (log2 domain)
//     l_h = sum_t 2^(s_ht - m_h)
//     U_h = sum_t 2^(s_ht - m_h) · K_t            (a full d-row, fp32)
// reduce_b.cu merges the partials and applies W_KV.
//
// Per CTA (one cluster of CL CTAs per work item; CTA r owns the columns
// [r·d/CL, (r+1)·d/CL) and the heads whose columns lie there):
//   warp 0      TMA producer: K tile = TT rows × (d/CL) columns, 128-byte
//               swizzled boxes of 16 rows × 64 columns, evict-first in L2.
//   warp 1      MMA issuer: Uᵀ (d-tile of 128 × heads) += K_tileᵀ · Pᵀ with
//               tcgen05.mma kind::f16 (A = K tile read MN-major, B = P
//               K-major), accumulator in TMEM: lane = d column, column = head.
//   warps 2..5  scores q_h·K_t (fp32 CUDA cores, 8 lanes per row and
//               shuffle reduction), online softmax with a lazy max (the
//               accumulator is rescaled in TMEM only when a head's max grows by
//               more than 2^8), P in bf16 to shared memory (and to the peer CTA
//               of the cluster through distributed shared memory), epilogue
//               TMEM -> partials in global memory.
// Every mbarrier wait is bounded; a timeout sets SLIM_DEV_TIMEOUT and the
// kernel drains its copies and MMAs, frees TMEM and returns.
#include <cuda_bf16.h>

#include "split_plan.cuh"

namespace slim {

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
  int n_slots;
  int stages;
  int npad;
  int min_rows;
  uint32_t tmem_cols;
  float scale_log2;
};

// Shared-memory carve-up, identical on host and device.
struct TCSmem {
  uint32_t k_off, p_off, alpha_off, bar_off, slot_off, plan_off, total;
};
__host__ __device__ inline TCSmem tc_smem_layout(int CL, int TT, int d, int npad, int stages, int B) {
  TCSmem s;
  const uint32_t dS = static_cast<uint32_t>(d / CL);
  uint32_t o = 0;
  s.k_off = o;
  o += static_cast<uint32_t>(stages) * TT * dS * 2u;
  s.p_off = o;
  o += static_cast<uint32_t>(stages) * npad * TT * 2u;
  s.alpha_off = o;
  o += static_cast<uint32_t>(stages) * npad * 4u;
  o = (o + 7u) & ~7u;
  s.bar_off = o;
  o += (5u * stages + 1u) * 8u;
  s.slot_off = o;
  o += 16u;
  s.plan_off = o;
  o += 3u * static_cast<uint32_t>(B + 1) * 4u;
  s.total = o + 1024u;  // slack for aligning the base to 1024 bytes
  return s;
}

template <int CL, int TT, int DHB, int HPW>
__global__ void __launch_bounds__(192, 1)
    decode_b_tc_kernel(const __grid_constant__ CUtensorMap kmap, const DecodeTCParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int DH = DHB * 64;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = (CL > 1) ? cluster_ctarank() : 0u;
  const uint32_t peer = rank ^ 1u;
  const int slot = blockIdx.x / CL;
  const int dS = p.d / CL, col0 = static_cast<int>(rank) * dS;
  const int ncb = dS / 64, ndt = dS / 128;
  const int H_own = p.H / CL, head0 = static_cast<int>(rank) * H_own;
  const int stages = p.stages, npad = p.npad;
  const TCSmem L = tc_smem_layout(CL, TT, p.d, npad, stages, p.B);
  uint8_t* kst = smem + L.k_off;
  uint8_t* pst = smem + L.p_off;
  float* alpha_s = reinterpret_cast<float*>(smem + L.alpha_off);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  uint64_t* full = bars;
  uint64_t* empty = bars + stages;
  uint64_t* pfull = bars + 2 * stages;
  uint64_t* pempty = bars + 3 * stages;
  uint64_t* corr = bars + 4 * stages;
  uint64_t* accfull = bars + 5 * stages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.slot_off);
  int* s_nb = reinterpret_cast<int*>(smem + L.plan_off);
  int* s_rows = s_nb + (p.B + 1);
  int* s_off = s_rows + (p.B + 1);
  const uint32_t kstage_bytes = static_cast<uint32_t>(TT) * dS * 2u;
  const uint32_t pstage_bytes = static_cast<uint32_t>(npad) * TT * 2u;

  pdl_launch_dependents();

  // ---------------------------------------------------------------- set-up
  if (warp == 0) {
    plan_split(p.lens, p.B, p.cap, p.append, p.n_slots, p.min_rows, s_nb, s_rows, s_off, p.ws_meta, p.status,
               blockIdx.x == 0);
    if (lane == 0) tma_prefetch_desc(&kmap);
  } else if (warp == 1) {
    if (lane == 0) {
      for (int s = 0; s < stages; ++s) {
        mbar_init(&full[s], 1);
        mbar_init(&empty[s], 1);
        mbar_init(&pfull[s], 4 * CL);
        mbar_init(&pempty[s], CL);
        mbar_init(&corr[s], 4);
      }
      mbar_init(accfull, 1);
      fence_barrier_init();
    }
    __syncwarp();
    tmem_alloc(tmem_slot, p.tmem_cols);
    tmem_relinquish();
  } else {
    // P buffers start at zero (padded heads stay zero); every alpha starts at 1.
    const int t = threadIdx.x - 64;
    uint32_t* pz = reinterpret_cast<uint32_t*>(pst);
    for (uint32_t i = t; i < stages * pstage_bytes / 4u; i += 128) pz[i] = 0u;
    for (int i = t; i < stages * npad; i += 128) alpha_s[i] = 1.0f;
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (CL > 1) cluster_sync();
  const uint32_t tmem = *tmem_slot;

  const SplitItem it = plan_lookup(slot, p.B, s_nb, s_rows, s_off);
  const int ntiles = (it.b >= 0) ? (it.row1 - it.row0 + TT - 1) / TT : 0;
  const int b = it.b;
  bool failed = false;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && ntiles > 0) {
      const uint64_t pol = l2_policy_evict_first();
      int issued = 0;
      for (int t = 0; t < ntiles; ++t) {
        const int s = t % stages;
        const uint32_t ph = static_cast<uint32_t>(t / stages) & 1u;
        if (t >= stages && !mbar_wait(&empty[s], ph ^ 1u, p.status)) {
          failed = true;
          break;
        }
        const int r_lo = it.row0 + t * TT;
        const int nbox = (min(TT, it.row1 - r_lo) + 15) / 16;
        mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(nbox) * 16u * 128u * ncb);
        const int y0 = static_cast<int>(static_cast<int64_t>(b) * p.cap + r_lo);
        uint8_t* dst = kst + s * kstage_bytes;
        for (int cb = 0; cb < ncb; ++cb)
          for (int rb = 0; rb < nbox; ++rb)
            tma_load_2d(dst + cb * TT * 128 + rb * 16 * 128, &kmap, col0 + cb * 64, y0 + rb * 16, &full[s], pol);
        issued = t + 1;
      }
      // drain: every issued copy must land before the CTA can exit
      for (int t = max(0, issued - stages); t < issued; ++t)
        mbar_wait(&full[t % stages], static_cast<uint32_t>(t / stages) & 1u, p.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && ntiles > 0) {
      const uint32_t idesc = idesc_bf16_f32(128, static_cast<uint32_t>(npad), 1u, 0u);
      const uint32_t kbase = smem_u32(kst), pbase = smem_u32(pst);
      for (int t = 0; t < ntiles; ++t) {
        const int s = t % stages;
        const uint32_t ph = static_cast<uint32_t>(t / stages) & 1u;
        if (!mbar_wait(&corr[s], ph, p.status) || !mbar_wait(&full[s], ph, p.status)) {
          failed = true;
          break;
        }
        tc_fence_after();
        const int r_lo = it.row0 + t * TT;
        const int nks = (min(TT, it.row1 - r_lo) + 15) / 16;
        const uint32_t ka = kbase + s * kstage_bytes, pa = pbase + s * pstage_bytes;
        for (int j = 0; j < ndt; ++j) {
          for (int kk = 0; kk < nks; ++kk) {
            const uint64_t ad = smem_desc(ka + (2 * j) * TT * 128 + kk * 16 * 128, TT * 128, 1024, kLayoutSW128);
            const uint64_t bd = smem_desc(pa + kk * 2 * 128, 128, (TT / 8) * 128, kLayoutNone);
            umma_f16(tmem + static_cast<uint32_t>(j * npad), ad, bd, idesc, (t > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(&empty[s]);
        if (CL > 1) umma_commit_mc(&pempty[s], static_cast<uint16_t>((1u << CL) - 1u));
        else umma_commit(&pempty[s]);
      }
      umma_commit(accfull);
      mbar_wait(accfull, 0, p.status);  // no MMA may be in flight at teardown
    }
  } else if (ntiles > 0) {
    // ------------------------------------------------------------ softmax warps
    const int sw = warp - 2;        // 0..3
    const int quarter = warp & 3;   // TMEM lane quarter this warp may access
    const int rr = lane >> 3, jj = lane & 7;
    float qr[HPW][DHB][8];
    float mref[HPW], lsum[HPW];
#pragma unroll
    for (int k = 0; k < HPW; ++k) {
      mref[k] = -INFINITY;
      lsum[k] = 0.f;
      const int hh = sw + 4 * k;
#pragma unroll
      for (int c = 0; c < DHB; ++c) {
        if (hh < H_own) {
          const float4* src =
              reinterpret_cast<const float4*>(p.q + static_cast<size_t>(b) * p.d + col0 + hh * DH + c * 64 + jj * 8);
          const float4 a0 = __ldg(src), a1 = __ldg(src + 1);
          qr[k][c][0] = a0.x; qr[k][c][1] = a0.y; qr[k][c][2] = a0.z; qr[k][c][3] = a0.w;
          qr[k][c][4] = a1.x; qr[k][c][5] = a1.y; qr[k][c][6] = a1.z; qr[k][c][7] = a1.w;
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) qr[k][c][e] = 0.f;
        }
      }
    }
    const int nb_old = it.nb - p.append;  // rows holding cached keys
    const uint32_t pst_base = smem_u32(pst);
    const uint32_t alpha_base = smem_u32(alpha_s);

    for (int t = 0; t < ntiles; ++t) {
      const int s = t % stages;
      const uint32_t ph = static_cast<uint32_t>(t / stages) & 1u;
      const int r_lo = it.row0 + t * TT;
      const int nvalid = min(TT, it.row1 - r_lo);
      const int nloaded = (nvalid + 15) & ~15;
      if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph, p.status))) { failed = true; break; }
      uint8_t* ks = kst + s * kstage_bytes;

      // Rows >= nb_old in this tile hold no cached key: the appended key goes
      // to row nb_old (also written to the cache), the rest become zero. Each
      // warp fixes the column blocks of its own heads, which are the only
      // columns it reads before the MMA (ordered by the proxy fence below).
      if (r_lo + nloaded > nb_old) {
        const int fr0 = max(nb_old - r_lo, 0);
#pragma unroll
        for (int k = 0; k < HPW; ++k) {
          const int hh = sw + 4 * k;
          if (hh >= H_own) continue;
#pragma unroll
          for (int c = 0; c < DHB; ++c) {
            const int cb = hh * DHB + c;
            for (int i = lane; i < (nloaded - fr0) * 8; i += 32) {
              const int row = fr0 + (i >> 3), j = i & 7;
              uint4 v = make_uint4(0u, 0u, 0u, 0u);
              if (p.append && r_lo + row == nb_old) {
                const size_t col = static_cast<size_t>(col0) + cb * 64 + j * 8;
                v = __ldg(reinterpret_cast<const uint4*>(p.k_new + static_cast<size_t>(b) * p.d + col));
                *reinterpret_cast<uint4*>(p.kcache + (static_cast<size_t>(b) * p.cap + nb_old) * p.d + col) = v;
              }
              *reinterpret_cast<uint4*>(ks + cb * TT * 128 + row * 128 + ((j ^ (row & 7)) << 4)) = v;
            }
          }
        }
        __syncwarp();
      }

      // P stage s is free once the MMAs that read it (tile t - stages) finished in every CTA.
      if (t >= stages && !__all_sync(0xffffffffu, mbar_wait(&pempty[s], ph ^ 1u, p.status))) {
        failed = true;
        break;
      }

      float alpha_k[HPW];
#pragma unroll
      for (int k = 0; k < HPW; ++k) {
        const int hh = sw + 4 * k;
        alpha_k[k] = 1.f;
        if (hh >= H_own) continue;
        float sv[TT / 4];
#pragma unroll
        for (int g = 0; g < TT / 4; ++g) {
          const int row = 4 * g + rr;
          float acc = 0.f;
#pragma unroll
          for (int c = 0; c < DHB; ++c) {
            const int cb = (hh * DH) / 64 + c;
            const uint4 v = *reinterpret_cast<const uint4*>(ks + cb * TT * 128 + row * 128 + ((jj ^ (row & 7)) << 4));
            acc = fmaf(qr[k][c][0], bf16lo(v.x), acc);
            acc = fmaf(qr[k][c][1], bf16hi(v.x), acc);
            acc = fmaf(qr[k][c][2], bf16lo(v.y), acc);
            acc = fmaf(qr[k][c][3], bf16hi(v.y), acc);
            acc = fmaf(qr[k][c][4], bf16lo(v.z), acc);
            acc = fmaf(qr[k][c][5], bf16hi(v.z), acc);
            acc = fmaf(qr[k][c][6], bf16lo(v.w), acc);
            acc = fmaf(qr[k][c][7], bf16hi(v.w), acc);
          }
          acc += __shfl_xor_sync(0xffffffffu, acc, 1);
          acc += __shfl_xor_sync(0xffffffffu, acc, 2);
          acc += __shfl_xor_sync(0xffffffffu, acc, 4);
          sv[g] = (row < nvalid) ? acc * p.scale_log2 : -INFINITY;
        }
        float mx = sv[0];
#pragma unroll
        for (int g = 1; g < TT / 4; ++g) mx = fmaxf(mx, sv[g]);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        if (t == 0) {
          mref[k] = mx;
        } else if (mx > mref[k] + 8.f) {
          alpha_k[k] = exp2f(mref[k] - mx);
          mref[k] = mx;
          lsum[k] *= alpha_k[k];
        }
        // lane (rr, jj) owns row 4*jj + rr of the tile
        float sel = sv[0];
#pragma unroll
        for (int g = 1; g < TT / 4; ++g) sel = (jj == g) ? sv[g] : sel;
        const int trow = 4 * jj + rr;
        if (jj < TT / 4) {
          const float pv = (trow < nvalid) ? exp2f(sel - mref[k]) : 0.f;
          const __nv_bfloat16 pb = __float2bfloat16_rn(pv);
          lsum[k] += __bfloat162float(pb);
          const int n = head0 + hh;
          const uint32_t off = static_cast<uint32_t>(s) * pstage_bytes +
                               static_cast<uint32_t>(((n >> 3) * (TT / 8) + (trow >> 3)) * 128 + (n & 7) * 16 +
                                                     (trow & 7) * 2);
          const uint16_t bits = __bfloat16_as_ushort(pb);
          asm volatile("st.shared.u16 [%0], %1;" ::"r"(pst_base + off), "h"(bits) : "memory");
          if (CL > 1) st_cluster_u16(mapa_shared(pst_base + off, peer), bits);
        }
        if (lane == 0) {
          const uint32_t aoff = static_cast<uint32_t>((s * npad + head0 + hh) * 4);
          alpha_s[s * npad + head0 + hh] = alpha_k[k];
          if (CL > 1) st_cluster_f32(mapa_shared(alpha_base + aoff, peer), alpha_k[k]);
        }
      }
      fence_proxy_async_smem();
      if (CL > 1) fence_proxy_async_cluster();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&pfull[s]);
        if (CL > 1) mbar_arrive_cluster(mapa_shared(smem_u32(&pfull[s]), peer));
      }

      // Lazy rescale: every CTA multiplies its TMEM columns of head n by the
      // alpha published for n, after the MMAs of the previous tile finished.
      if (!__all_sync(0xffffffffu, mbar_wait(&pfull[s], ph, p.status))) { failed = true; break; }
      const float my_alpha = (lane < npad) ? alpha_s[s * npad + lane] : 1.f;
      if (t > 0 && __any_sync(0xffffffffu, my_alpha != 1.f)) {
        const int sp = (t - 1) % stages;
        const uint32_t php = static_cast<uint32_t>((t - 1) / stages) & 1u;
        if (!__all_sync(0xffffffffu, mbar_wait(&empty[sp], php, p.status))) { failed = true; break; }
        tc_fence_after();
        for (int j = 0; j < ndt; ++j) {
          for (int c16 = 0; c16 < npad; c16 += 16) {
            const uint32_t ta = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + j * npad + c16;
            float v[16];
            tmem_ld16(ta, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] *= __shfl_sync(0xffffffffu, my_alpha, (c16 + i) & 31);
            tmem_st16(ta, v);
          }
        }
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&corr[s]);
    }

    // ------------------------------------------------------------ epilogue
    if (!failed && __all_sync(0xffffffffu, mbar_wait(accfull, 0, p.status))) {
      tc_fence_after();
      const size_t item = static_cast<size_t>(slot);
      for (int j = 0; j < ndt; ++j) {
        for (int c16 = 0; c16 < npad; c16 += 16) {
          float v[16];
          tmem_ld16(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + j * npad + c16, v);
          tmem_wait_ld();
          const int dcol = col0 + j * 128 + quarter * 32 + lane;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int n = c16 + i;
            if (n < p.H) p.ws_U[(item * p.H + n) * p.d + dcol] = v[i];
          }
        }
      }
#pragma unroll
      for (int k = 0; k < HPW; ++k) {
        const int hh = sw + 4 * k;
        const float tot = warp_sum(lsum[k]);
        if (hh < H_own && lane == 0) {
          p.ws_m[item * p.H + head0 + hh] = mref[k];
          p.ws_l[item * p.H + head0 + hh] = tot;
        }
      }
    }
  }

  // ---------------------------------------------------------------- teardown
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
  int CL, TT, DHB, HPW, stages, npad;
  uint32_t tmem_cols, smem;
};

uint32_t pow2_cols(uint32_t c) {
  uint32_t r = 32;
  while (r < c) r <<= 1;
  return r;
}

// Template instances compiled below (CL, TT, DHB, HPW); pick_config only returns these.
#define SLIM_TC_INSTANCES(X)                                                                          \
  X(1, 32, 1, 2) X(1, 32, 1, 4) X(1, 32, 1, 5) X(1, 32, 1, 8) X(1, 16, 1, 2) X(1, 16, 1, 4) X(1, 16, 1, 5) \
  X(1, 16, 1, 8) X(1, 32, 2, 2) X(1, 32, 2, 4) X(1, 16, 2, 2) X(1, 16, 2, 4) X(2, 32, 1, 2) X(2, 32, 1, 4) \
  X(2, 16, 1, 2) X(2, 16, 1, 4) X(2, 16, 1, 8) X(2, 32, 2, 2) X(2, 32, 2, 4) X(2, 16, 2, 2) X(2, 16, 2, 4)

bool tc_instantiated(int CL, int TT, int DHB, int HPW) {
#define SLIM_TC_MATCH(a, b, c, e) if (CL == a && TT == b && DHB == c && HPW == e) return true;
  SLIM_TC_INSTANCES(SLIM_TC_MATCH)
#undef SLIM_TC_MATCH
  return false;
}

bool pick_config(int B, int d, int H, TCConfig* out) {
  if (H <= 0 || d % H) return false;
  const int dh = d / H;
  if (dh != 64 && dh != 128) return false;
  const int smem_cap = max_smem_optin();
  const int npad = ((H + 15) / 16) * 16;
  for (int CL = 1; CL <= 2; ++CL) {
    if (d % (128 * CL) || H % CL || (d / CL) % dh) continue;
    const int H_own = H / CL;
    const int hpw = (H_own + 3) / 4;
    int HPW = hpw <= 2 ? 2 : hpw <= 4 ? 4 : hpw <= 5 ? 5 : hpw <= 8 ? 8 : 0;
    if (!HPW) continue;
    if (npad > 32) continue;
    const uint32_t cols = static_cast<uint32_t>((d / CL / 128) * npad);
    if (cols > 512) continue;
    for (int TT : {32, 16}) {
      int stages = 0;
      for (int s = 8; s >= 2; --s) {
        if (tc_smem_layout(CL, TT, d, npad, s, B).total <= static_cast<uint32_t>(smem_cap)) {
          stages = s;
          break;
        }
      }
      if (stages == 0) continue;
      if (TT == 32 && stages < 3) continue;  // prefer more stages of 16 rows
      if (!tc_instantiated(CL, TT, dh / 64, HPW)) continue;
      out->CL = CL;
      out->TT = TT;
      out->DHB = dh / 64;
      out->HPW = HPW;
      out->stages = stages;
      out->npad = npad;
      out->tmem_cols = pow2_cols(cols);
      out->smem = tc_smem_layout(CL, TT, d, npad, stages, B).total;
      return true;
    }
  }
  return false;
}

template <int CL, int TT, int DHB, int HPW>
cudaError_t launch_tc(const CUtensorMap& map, const DecodeTCParams& prm, const TCConfig& c, cudaStream_t st) {
  auto kern = decode_b_tc_kernel<CL, TT, DHB, HPW>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(c.smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(prm.n_slots * CL), 1, 1);
  cfg.blockDim = dim3(192, 1, 1);
  cfg.dynamicSmemBytes = c.smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, map, prm);
}

}  // namespace

bool decode_b_tc_supported(int B, int d, int H) {
  TCConfig c;
  return pick_config(B, d, H, &c);
}

cudaError_t launch_decode_b_tc(const DecodeArgs& a, const SplitWorkspace& ws, cudaStream_t st, int* launches) {
  TCConfig c;
  if (a.dtype != SLIM_BF16 || !pick_config(a.B, a.d, a.H, &c)) return cudaErrorNotSupported;
  CUtensorMap map;
  if (!encode_tmap_2d_bf16(&map, a.kcache, static_cast<uint64_t>(a.d), static_cast<uint64_t>(a.B) * a.cap,
                           static_cast<uint64_t>(a.d) * 2u, 64, 16, true))
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
  prm.n_slots = max(num_sms() / c.CL, a.B);
  if (prm.n_slots > ws.max_items) return cudaErrorInvalidValue;
  prm.stages = c.stages;
  prm.npad = c.npad;
  prm.min_rows = max(16, 8 * a.H);
  prm.tmem_cols = c.tmem_cols;
  prm.scale_log2 = 1.4426950408889634f / sqrtf(static_cast<float>(a.d / a.H));
  cudaError_t e = cudaErrorNotSupported;
#define SLIM_TC_CASE(CL_, TT_, DHB_, HPW_)                                                  \
  if (c.CL == CL_ && c.TT == TT_ && c.DHB == DHB_ && c.HPW == HPW_) {                        \
    e = launch_tc<CL_, TT_, DHB_, HPW_>(map, prm, c, st);                                    \
  } else
  SLIM_TC_INSTANCES(SLIM_TC_CASE)
  { e = cudaErrorNotSupported; }
#undef SLIM_TC_CASE
  if (e == cudaSuccess && launches) ++*launches;
  return e;
}

}  // namespace slim
