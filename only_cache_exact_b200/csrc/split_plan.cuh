// Split-T work list for the decode kernels ("flash-decoding" with contiguous
// shares, as in stream-K GEMM scheduling): the attended rows of every
// sequence, in 16-row units, are laid end to end on one line, and the line is
// cut into G equal contiguous shares, one per work group (a CTA or a CTA
// cluster). Group g reduces the rows of its share to one softmax partial per
// sequence the share touches (a "segment"), so every group streams the same
// number of rows whatever the mix of lengths, and a sequence has only as many
// partials as groups overlap it. Each non-empty sequence is preceded on the
// line by kSegCostUnits extra units that stand for the fixed cost of starting
// a partial, so a share that covers the start of a sequence takes fewer rows.
// Every CTA of a split kernel computes the same plan from `lens`, so no
// pre-pass kernel is needed.
#pragma once

#include "ptx.cuh"

namespace slim {

// Line units charged for starting a partial (a pipeline restart and an epilogue).
constexpr int kSegCostUnits = 4;

struct SplitItem {
  int b;     // sequence
  int row0;  // first row of the segment within the sequence
  int row1;  // one past the last row
  int nb;    // attended rows of the sequence (incl. the appended one)
  int slot;  // partial slot of the segment in the workspace
};

// Group g's share is [floor(g·T/G), floor((g+1)·T/G)) of the T line units.
__device__ __forceinline__ unsigned lean_start(int g, unsigned total, int G) {
  return static_cast<unsigned>((static_cast<unsigned long long>(g) * total) / static_cast<unsigned>(G));
}
// The group whose share contains line unit x (x < T).
__device__ __forceinline__ int lean_group_of(unsigned x, unsigned total, int G) {
  return static_cast<int>(((static_cast<unsigned long long>(x) + 1ull) * static_cast<unsigned>(G) - 1ull) / total);
}

// Exclusive prefix sum over [0, B) of v(b) by ONE warp into dst[0..B]; returns the total.
template <typename F>
__device__ __forceinline__ unsigned warp_scan_excl(int B, unsigned* dst, F v) {
  const int lane = threadIdx.x & 31;
  unsigned carry = 0;
  for (int base = 0; base < B; base += 32) {
    const int b = base + lane;
    const unsigned c = b < B ? v(b) : 0u;
    unsigned x = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (b < B) dst[b] = carry + x - c;
    carry += __shfl_sync(0xffffffffu, x, 31);
  }
  if (lane == 0) dst[B] = carry;
  __syncwarp();
  return carry;
}

// Run by ONE full warp. B work sequences; sequence b reads its length from lens[b / rep] (rep > 1
// when several work sequences share one cache sequence, e.g. one per group of heads). Shared
// arrays: s_nb [B] attended rows, s_q [B+1] line offset of every sequence, s_soff [B+1] first
// partial slot of every sequence, s_plan [2] = {T, G}.
// n_groups work groups are launched; fewer take work when the rows do not give each group at
// least min_rows (a partial costs H·d·4 bytes to write and merge).
// report != 0: also writes the merge metadata and ORs length errors into *status.
// Work-list metadata for the merge kernels:
//   meta[0]          total number of partial slots
//   meta[1 + b]      first slot of sequence b (b = 0..B), meta[1 + B] = total
//   meta[2 + B + b]  flags of sequence b (kSeqAppend: lens[b] must advance by one)
__device__ inline void plan_lean(const int32_t* __restrict__ lens, int B, int rep, int64_t cap, int append,
                                 int n_groups, int min_rows, int* s_nb, unsigned* s_q, unsigned* s_soff,
                                 unsigned* s_plan, int32_t* meta, int32_t* status, bool report) {
  const int lane = threadIdx.x & 31;
  int bad = 0;
  unsigned R = 0;
  for (int b = lane; b < B; b += 32) {
    const int L = __ldcg(lens + b / rep);
    int nb;
    if (L < 0 || static_cast<int64_t>(L) > cap) {
      nb = 0;
      bad |= SLIM_DEV_BADLEN;
    } else if (append && static_cast<int64_t>(L) >= cap) {
      nb = 0;
      bad |= SLIM_DEV_OVERFLOW;
    } else {
      nb = L + append;
    }
    s_nb[b] = nb;
    R += static_cast<unsigned>(nb);
    if (report) meta[2 + B + b] = (nb > 0 && append) ? kSeqAppend : 0;
  }
  // attended rows fit in 31 bits (B * cap < 2^31), so single-instruction warp reductions suffice
  R = __reduce_add_sync(0xffffffffu, R);
  bad = __reduce_or_sync(0xffffffffu, bad);
  if (report && lane == 0 && bad) atomicOr(status, bad);
  __syncwarp();
  const unsigned total = warp_scan_excl(B, s_q, [&](int b) {
    const int nb = s_nb[b];
    return nb > 0 ? static_cast<unsigned>((nb + 15) >> 4) + kSegCostUnits : 0u;
  });
  int G = n_groups;
  const unsigned mr = static_cast<unsigned>(max(min_rows, 16));
  if (R < mr * static_cast<unsigned>(G)) G = max(1, static_cast<int>(R / mr));
  const unsigned T = max(total, 1u);
  const unsigned slots = warp_scan_excl(B, s_soff, [&](int b) {
    if (s_nb[b] <= 0) return 0u;
    const unsigned rs = s_q[b] + kSegCostUnits, re = s_q[b + 1];
    return static_cast<unsigned>(lean_group_of(re - 1u, T, G) - lean_group_of(rs, T, G) + 1);
  });
  if (lane == 0) {
    s_plan[0] = total;
    s_plan[1] = static_cast<unsigned>(G);
  }
  if (report) {
    for (int b = lane; b <= B; b += 32) meta[1 + b] = static_cast<int32_t>(s_soff[b]);
    if (lane == 0) meta[0] = static_cast<int32_t>(slots);
  }
  __syncwarp();
}

// The segments of one group, in line order (any thread; every role of a CTA walks the same list).
struct LeanCursor {
  int g, b, B;
  unsigned x0, x1, T;
  int G;

  __device__ void init(int group, int B_, const unsigned* s_q, const unsigned* s_plan) {
    g = group;
    B = B_;
    T = s_plan[0];
    G = static_cast<int>(s_plan[1]);
    b = B;
    x0 = x1 = 0;
    if (g >= G || T == 0) return;
    x0 = lean_start(g, T, G);
    x1 = lean_start(g + 1, T, G);
    int lo = 0, hi = B;  // largest b with s_q[b] <= x0
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s_q[mid] <= x0) lo = mid; else hi = mid;
    }
    b = lo;
  }

  __device__ bool next(SplitItem& it, const int* s_nb, const unsigned* s_q, const unsigned* s_soff) {
    while (b < B && s_q[b] < x1) {
      const int bb = b++;
      const int nb = s_nb[bb];
      if (nb <= 0) continue;
      const unsigned rs = s_q[bb] + kSegCostUnits, re = s_q[bb + 1];
      const unsigned lo = max(x0, rs), hi = min(x1, re);
      if (lo >= hi) continue;
      it.b = bb;
      it.nb = nb;
      it.row0 = static_cast<int>(lo - rs) * 16;
      it.row1 = min(static_cast<int>(hi - rs) * 16, nb);
      it.slot = static_cast<int>(s_soff[bb]) + (g - lean_group_of(rs, T, G));
      return true;
    }
    return false;
  }
};

}  // namespace slim
