// Internal declarations shared by the libslim translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/slim.h"

namespace slim {

// A wait on an mbarrier gives up after this long (global timer, ns).
constexpr uint64_t kWaitLimitNs = 1000000000ull;

// Work-list metadata written by the split kernel for the merge kernel:
//   meta[0]          total number of partial slots
//   meta[1 + b]      first slot of sequence b (b = 0..B), meta[1 + B] = total
//   meta[2 + B + b]  flags of sequence b (kSeqAppend: lens[b] must advance by one)
constexpr int kSeqAppend = 1;
__host__ __device__ inline size_t meta_ints(int B) { return static_cast<size_t>(2 * B + 2); }

// Scratch of the split-T orderings, carved from the caller's workspace.
struct SplitWorkspace {
  float* U;      // (b): [slots][H][d] unnormalised softmax·K rows;  (a): [slots][d] softmax·V
  float* m;      // [slots][H] running max (log2 domain)
  float* l;      // [slots][H] softmax denominators relative to m
  int32_t* meta; // meta_ints(B)
  void* vbuf;    // (a) only: [B][cap][d] materialised V = K·W_KV
  void* qstage;  // staging for slim_decode_step_host: q, k_new, out
  int max_items;
};

struct DecodeArgs {
  const float* q;
  const void* k_new;
  void* kcache;
  int32_t* lens;
  const void* w_kv;
  int dtype, B, d, H;
  int64_t cap;
  float* out;
  int32_t* status;
  uint64_t wait_ns = 0;  // 0: kWaitLimitNs
  int stall = 0;         // test hook (slim_debug_stall_next)
};

// ---- launchers (return cudaError_t of the launch) ----
// Variant (b), tcgen05 path (bf16). Returns cudaErrorNotSupported if the shape has no tcgen05 config.
cudaError_t launch_decode_b_tc(const DecodeArgs& a, const SplitWorkspace& ws, cudaStream_t st, int* launches);
bool decode_b_tc_supported(int B, int d, int H);
// Cluster size of the tcgen05 split kernel for this shape (0: no tcgen05 configuration).
int decode_b_tc_cluster(int B, int d, int H);
// Variant (b), CUDA-core path (fp32 or bf16 cache).
cudaError_t launch_decode_b_simt(const DecodeArgs& a, const SplitWorkspace& ws, cudaStream_t st, int* launches);
bool decode_b_simt_supported(int B, int d, int H);
// Merge of variant (b) partials and the W_KV projection; advances lens.
cudaError_t launch_reduce_b(const DecodeArgs& a, const SplitWorkspace& ws, bool pdl, cudaStream_t st,
                            int* launches);
// Variant (a) on tensor cores: V tiles made in TMEM and used there (V never in global memory).
bool decode_a_tc_supported(int dtype, int B, int d, int H);
size_t decode_a_tc_slots(int B, int d, int64_t cap);  // tile partials its workspace must hold
cudaError_t launch_decode_a_tc(const DecodeArgs& a, const SplitWorkspace& ws, cudaStream_t st, int* launches);
// Variant (a): append, V = K·W_KV, split flash-decode over K and V, merge (the tcgen05 path above
// where supported).
cudaError_t launch_decode_a(const DecodeArgs& a, const SplitWorkspace& ws, cudaStream_t st, int* launches);
bool decode_a_supported(int dtype, int B, int d, int H);
// Prompt-phase projection K = X·W_K into the cache at lens[b]; then lens += n.
cudaError_t launch_prefill(const void* X, const void* W, void* kcache, int32_t* lens, int dtype, int B, int n, int d,
                           int64_t cap, int32_t* status, cudaStream_t st, int* launches);
cudaError_t launch_reduce_a(const DecodeArgs& a, const SplitWorkspace& ws, cudaStream_t st, int* launches);
// Row-wise GEMM used by variant (a): Y[b][t] = K[b][t]·W for t < lens[b] (+append) rows of each sequence.
// _any picks the tcgen05 kernel for bf16 shapes it supports, else the CUDA-core one.
cudaError_t launch_rows_gemm_any(const void* A, const void* W, void* Y, const int32_t* lens, int rows_extra,
                                 int dtype, int B, int d, int64_t cap, int32_t* status, cudaStream_t st,
                                 int* launches);
cudaError_t launch_rows_gemm(const void* A, const void* W, void* Y, const int32_t* lens, int rows_extra, int dtype,
                             int B, int d, int64_t cap, cudaStream_t st, int* launches);

// Standard MHA decode over explicit K and V caches (the comparison baseline), bf16.
bool decode_kv_supported(int B, int d, int H, int64_t cap);
size_t kv_ws_slots(int B, int d);  // partial slots its workspace needs
cudaError_t launch_decode_kv(const float* q, const void* k_new, const void* v_new, void* kcache, void* vcache,
                             int32_t* lens, int B, int d, int H, int64_t cap, float* out, float* wsO, float* wsm,
                             float* wsl, int32_t* meta, int32_t* status, cudaStream_t st, int* launches);

// Prompt-phase attention output: causal attention of the n prompt queries over the K-only cache
// with V = K·W_KV materialised once (ordering (a)).
bool prefill_attn_supported(int dtype, int d, int H);
cudaError_t launch_prefill_attn(const void* Q, const void* kcache, const void* vbuf, const int32_t* lens, int B,
                                int n, int d, int H, int64_t cap, float* out, int32_t* status, cudaStream_t st,
                                int* launches);
cudaError_t launch_rows_gemm_tc(const void* A, const void* W, void* Y, const int32_t* lens, int rows_extra, int B,
                                int d, int64_t cap, int32_t* status, cudaStream_t st, int* launches);

// Step front end: q = x·W_Q (fp32) and, with W_K, k = x·W_K (cache dtype) for B input rows.
bool front_tc_supported(int dtype, int d);
int front_tc_split(int d, bool with_k);  // cluster size of the tcgen05 front end
cudaError_t launch_front(const void* x, const void* W_Q, const void* W_K, float* q, void* k, int dtype, int B, int d,
                         int32_t* status, cudaStream_t st, int* launches);

// Tensor map encoding through the driver entry point (no link-time libcuda dependency).
bool encode_tmap_2d_bf16(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                         uint32_t box_inner, uint32_t box_outer, bool swizzle128);

// General 3-D bf16 tiled map: dims {d0, d1, d2} (d0 innermost, contiguous), byte strides s1, s2 of
// dims 1 and 2, box {b0, b1, b2}, 128-byte swizzle (b0 * 2 must be <= 128).
bool encode_tmap_3d_bf16(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1,
                         uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2);
// Tiled map of any rank <= 5: dims (innermost first), byte strides of dims 1.., box; no
// interleave, optional 128-byte swizzle, zero fill out of range.
bool encode_tmap(CUtensorMap* map, CUtensorMapDataType type, int rank, const void* base, const uint64_t* dims,
                 const uint64_t* strides, const uint32_t* box, bool swizzle128);
// K cache [rows][d] bf16 as a 3-D map {64 columns, rows, d/64 column blocks} with a box of
// 64 x 16 x box_blocks, 128-byte swizzle: one load brings 16 rows of box_blocks column blocks.
bool encode_tmap_kslab(CUtensorMap* map, const void* base, uint64_t rows, int d, int box_blocks);

int num_sms();
int max_smem_optin();

}  // namespace slim
