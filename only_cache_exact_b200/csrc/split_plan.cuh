// Split-T work list for the decode kernels ("flash-decoding" style): the
// attended rows of every sequence are cut into row chunks so that the total
// number of chunks fills the launched work slots, then each slot (a CTA or a
// CTA cluster) reduces one chunk to a softmax partial. Every CTA of a split
// kernel computes the same plan from `lens`, so no pre-pass kernel is needed.
#pragma once

#include "ptx.cuh"

namespace slim {

struct SplitItem {
  int b;     // sequence, -1 if this slot has no work
  int row0;  // first row of the chunk within the sequence
  int row1;  // one past the last row
  int nb;    // attended rows of the sequence (incl. the appended one)
};

// Smallest chunk length C (a multiple of 16 rows, at least min_rows) such that
// cutting every sequence into ceil(nb / C) chunks needs at most n_slots work
// items. Bracketed first: C >= R / n_slots is necessary, and
// C >= R / (n_slots - nonempty) is sufficient (ceil adds at most one chunk per
// sequence), so the binary search usually runs a handful of steps. One warp.
// All quantities fit in 32 bits (R = attended rows < 2^31): the divisions stay
// 32-bit, which keeps this dependent chain short.
__device__ inline int plan_chunk(const int* s_nb, int B, unsigned n_slots, int min_rows, unsigned R, int nonempty,
                                 int max_nb) {
  const int lane = threadIdx.x & 31;
  const int cap16 = max((max_nb + 15) >> 4, 1);
  int lo = (max(min_rows, 16) + 15) >> 4;
  lo = max(lo, static_cast<int>((R + 16u * n_slots - 1u) / (16u * n_slots)));  // ceil(R / (16 n_slots))
  int hi = cap16;
  if (n_slots > static_cast<unsigned>(nonempty)) {
    const unsigned free_slots = n_slots - static_cast<unsigned>(nonempty);
    hi = min(hi, static_cast<int>((R + 16u * free_slots - 1u) / (16u * free_slots)));
  }
  if (lo >= hi) return max(lo, 1) << 4;
#pragma unroll 1
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    const int C = mid << 4;
    int cnt = 0;
    for (int b = lane; b < B; b += 32) cnt += static_cast<int>((static_cast<unsigned>(s_nb[b]) + C - 1) / C);
    cnt = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(cnt)));
    if (static_cast<unsigned>(cnt) <= n_slots) hi = mid; else lo = mid + 1;
  }
  return lo << 4;
}

// Run by ONE full warp. s_nb, s_rows: [B]; s_off: [B+1] (shared memory).
// The work items are processed by n_groups CTA groups (CTAs or clusters),
// group c taking items c, c + n_groups, ...; up to max_items items in total
// (max_items >= B). The number of items per group is chosen among powers of
// two to minimise the estimated longest group (rows of its items plus a fixed
// per-item cost), which balances ragged batches.
// report != 0: also writes the merge metadata and ORs length errors into *status.
__device__ inline void plan_split(const int32_t* __restrict__ lens, int B, int64_t cap, int append, int n_groups,
                                  int max_items, int min_rows, int* s_nb, int* s_rows, int* s_off, int32_t* meta,
                                  int32_t* status, bool report) {
  const int lane = threadIdx.x & 31;
  // one slot group per item (a single candidate k below): the previous plan's chunk is read with
  // the lengths and tried first
  const bool single_k = 2LL * n_groups > max_items || max(2 * n_groups, B) > max_items;
  const int hint = single_k ? __ldcg(meta + 2 + 2 * B) : 0;
  int bad = 0, nonempty = 0, max_nb = 0;
  long long R = 0;
  for (int b = lane; b < B; b += 32) {
    const int L = __ldcg(lens + b);
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
    R += nb;
    nonempty += nb > 0;
    max_nb = max(max_nb, nb);
    if (report) meta[2 + B + b] = (nb > 0 && append) ? kSeqAppend : 0;
  }
  // attended rows fit in 31 bits (B * cap < 2^31), so single-instruction warp reductions suffice
  R = static_cast<long long>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(R)));
  nonempty = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(nonempty)));
  max_nb = __reduce_max_sync(0xffffffffu, max_nb);
  bad = __reduce_or_sync(0xffffffffu, bad);
  if (report && lane == 0 && bad) atomicOr(status, bad);
  __syncwarp();

  // Fast path: the chunk the previous plan on this workspace chose is the answer again when it
  // is still the smallest feasible one, i.e. it fits n_slots and 16 rows less does not (or is
  // below the lower bound). Lengths usually grow by one row per step, so it rarely changes.
  const unsigned n1 = static_cast<unsigned>(max(n_groups, nonempty));
  const int lo16 = max((max(min_rows, 16) + 15) >> 4,
                       static_cast<int>((static_cast<unsigned>(R) + 16u * n1 - 1u) / (16u * n1)));
  bool fast = false;
  if (single_k && hint >= 16 && (hint & 15) == 0 && (hint >> 4) >= lo16 && hint <= max(max_nb, 16) + 16) {
    unsigned c0 = 0, c1 = 0;
    const unsigned C0 = static_cast<unsigned>(hint), C1 = C0 - 16u;
    for (int b = lane; b < B; b += 32) {
      const unsigned nb = static_cast<unsigned>(s_nb[b]);
      c0 += (nb + C0 - 1u) / C0;
      if (C1 > 0u) c1 += (nb + C1 - 1u) / C1;
    }
    c0 = __reduce_add_sync(0xffffffffu, c0);
    c1 = __reduce_add_sync(0xffffffffu, c1);
    fast = c0 <= n1 && ((hint >> 4) == lo16 || c1 > n1);
  }
  constexpr long long kItemCostRows = 128;  // epilogue + pipeline restart, in K rows
  int chunk = fast ? hint : 16;
  long long best = fast ? 0 : -1;
  for (int k = 1; !fast && (static_cast<long long>(k) * n_groups <= max_items || k == 1); k <<= 1) {
    const unsigned n_slots = static_cast<unsigned>(max(k * n_groups, nonempty));
    if (n_slots > static_cast<unsigned>(max_items) && k > 1) break;
    const int C = plan_chunk(s_nb, B, n_slots, min_rows, static_cast<unsigned>(R), nonempty, max_nb);
    int items = 0;
    for (int b = lane; b < B; b += 32) items += static_cast<int>((static_cast<unsigned>(s_nb[b]) + C - 1) / C);
    items = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(items)));
    const long long per_group = static_cast<long long>((static_cast<unsigned>(items) + n_groups - 1) / n_groups);
    const long long est = per_group * (C + kItemCostRows);
    if (best < 0 || est < best) {
      best = est;
      chunk = C;
    }
    if (k > 64) break;
  }

  int carry = 0;
  for (int base = 0; base < B; base += 32) {
    const int b = base + lane;
    int c = 0;
    if (b < B) {
      const int nb = s_nb[b];
      s_rows[b] = chunk;
      if (nb > 0) c = static_cast<int>((static_cast<unsigned>(nb) + chunk - 1) / chunk);
    }
    int x = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (b < B) s_off[b] = carry + x - c;
    carry += __shfl_sync(0xffffffffu, x, 31);
  }
  if (lane == 0) s_off[B] = carry;
  __syncwarp();
  if (report) {
    for (int b = lane; b <= B; b += 32) meta[1 + b] = s_off[b];
    if (lane == 0) {
      meta[0] = carry;
      meta[2 + 2 * B] = chunk;
    }
  }
}

// Work item of slot `slot` from a finished plan (any thread).
__device__ inline SplitItem plan_lookup(int slot, int B, const int* s_nb, const int* s_rows, const int* s_off) {
  SplitItem it{-1, 0, 0, 0};
  if (slot >= s_off[B]) return it;
  int lo = 0, hi = B;  // largest b with s_off[b] <= slot
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_off[mid] <= slot) lo = mid; else hi = mid;
  }
  // skip empty sequences sharing the same offset
  int b = lo;
  while (b < B && s_off[b + 1] <= slot) ++b;
  const int c = slot - s_off[b];
  it.b = b;
  it.nb = s_nb[b];
  it.row0 = c * s_rows[b];
  it.row1 = min(it.row0 + s_rows[b], it.nb);
  return it;
}

}  // namespace slim
