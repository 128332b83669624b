/*
 * slim.h — C ABI of libslim.so: the generation-phase (decode) step of Slim
 * attention over a K-only context cache, and the prompt-phase K projection
 * that fills that cache, on NVIDIA B200 (sm_100a).
 *
 * Method (Slim Attention article, section "K-Cache is All You Need"): in
 * multi-head attention with square projections, W_K invertible gives
 * W_KV = W_K^(-1)·W_V and V = X·W_V = K·W_KV, so only K is cached and the
 * values are recomputed from it. A generation step forms the scores of q
 * against the cached K, takes the per-head softmax, and either
 *   (a) computes V = K·W_KV and multiplies the softmax by V, or
 *   (b) multiplies the softmax by K first and that d-vector by W_KV,
 *       which the article calls cheaper for long sequences;
 * finally this step's k is appended to the K cache.
 *
 * Conventions (readings where the pages are silent):
 *   - row vectors: K = X·W_K, all matrices d×d row-major;
 *   - head h owns columns [h·d_h, (h+1)·d_h), d_h = d/H, softmax scale 1/sqrt(d_h);
 *   - a step appends its k before attending, so it attends to its own key;
 *   - the output is the concatenation of head outputs (no W_O, no residual).
 *
 * Memory: every pointer argument is a DEVICE pointer owned by the caller,
 * except where a name ends in _host. The library allocates no device memory;
 * scratch comes from the caller's `workspace`. All calls are asynchronous on
 * `stream` (a cudaStream_t, NULL = legacy default stream) unless stated.
 *
 * K cache layout: [B][cap][d] row-major in the cache dtype; sequence b's
 * valid rows are 0..lens[b]-1. `lens` is a device int32[B] updated in place
 * by the calls that append, so repeated calls (and CUDA-graph replays) advance.
 *
 * Errors: host-detected problems return a negative SLIM_E* code and launch
 * nothing. Problems only visible on the device (lengths) are OR-ed as
 * SLIM_DEV_* bits into the caller's device int32 `*dev_status`, which is
 * never cleared by the library; the offending sequence is skipped and its
 * output row set to zero. Kernels never trap. Every internal wait is bounded:
 * SLIM_DEV_TIMEOUT reports one that gave up.
 */
#ifndef SLIM_H_
#define SLIM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes. */
#define SLIM_OK 0
#define SLIM_EINVAL (-1)       /* null pointer, bad size, d % H != 0, bad dtype/variant */
#define SLIM_EWORKSPACE (-2)   /* workspace null, too small or not 256-byte aligned */
#define SLIM_ECUDA (-3)        /* a CUDA runtime call or launch failed */
#define SLIM_EUNSUPPORTED (-4) /* valid arguments this build has no kernel for */

/* Device status bits (OR-ed into *dev_status). */
#define SLIM_DEV_OVERFLOW 1 /* appending would exceed cap: sequence skipped, lens unchanged */
#define SLIM_DEV_BADLEN 2   /* lens[b] < 0 or lens[b] > cap: sequence skipped */
#define SLIM_DEV_TIMEOUT 4  /* a bounded in-kernel wait gave up (internal error) */

/* Cache / weight element types. */
#define SLIM_F32 0  /* fp32 storage, fp32 arithmetic */
#define SLIM_BF16 1 /* bf16 storage, fp32 accumulation (tensor cores where the work is a contraction) */

/* Decode orderings (section "K-Cache is All You Need", generation phase). */
#define SLIM_AUTO 0      /* pick (a) or (b) from the measured table (slim_tune), default (b) */
#define SLIM_VARIANT_A 1 /* materialise V = K·W_KV, then softmax·V */
#define SLIM_VARIANT_B 2 /* softmax·K first, then ·W_KV */

/*
 * slim_prefill_k — prompt phase: K = X·W_K for n new tokens per sequence,
 * written to rows lens[b] .. lens[b]+n-1 of the cache; then lens[b] += n.
 * Source: section "K-Cache is All You Need", prompt phase (Q and K of all
 * prompt tokens in parallel; K is cached, V is not computed).
 *
 *   X       [B][n][d] in `dtype`            (device, read)
 *   W_K     [d][d]    in `dtype`            (device, read)
 *   Kcache  [B][cap][d] in `dtype`          (device, rows written)
 *   lens    int32[B]                        (device, read then += n)
 *   dtype   SLIM_BF16: tcgen05 GEMM, fp32 accumulation, bf16 round-to-nearest
 *           output; SLIM_F32: one fp32 accumulator per output, k ascending,
 *           fused multiply-add per step (bitwise reproducible).
 *   B, n, d n >= 1, d >= 1; SLIM_BF16 needs d % 256 == 0.
 *   cap     rows per sequence in the cache (>= 1)
 *   dev_status  device int32 (SLIM_DEV_* bits); a sequence with
 *           lens[b] + n > cap is skipped with SLIM_DEV_OVERFLOW.
 */
int slim_prefill_k(const void* X, const void* W_K, void* Kcache, int32_t* lens, int dtype, int B, int n, int d,
                   int64_t cap, int32_t* dev_status, void* stream);

/*
 * slim_decode_workspace_bytes — device scratch needed by slim_decode_step /
 * slim_decode_step_host for these sizes on the current device (0 on bad
 * arguments). The caller allocates it (256-byte aligned) and may reuse it
 * for every call with the same or smaller sizes; calls sharing one
 * workspace must not overlap on the GPU.
 */
size_t slim_decode_workspace_bytes(int dtype, int B, int d, int H, int64_t cap, int variant);

/*
 * slim_decode_step — one generation step for B independent sequences.
 * Source: section "K-Cache is All You Need", generation phase (scores of q
 * against the cached K, softmax, V = K·W_KV by ordering (a) or (b), append k).
 *
 *   q       float[B][d]          this step's queries (device, read)
 *   k_new   [B][d] in `dtype`    this step's keys, appended at row lens[b]
 *           before attending; NULL = no append (cross-attention over a
 *           fixed cache: attend over lens[b] rows, lens unchanged)
 *   Kcache  [B][cap][d] `dtype`  (device; row lens[b] written when appending)
 *   lens    int32[B]             (device; += 1 per appended sequence)
 *   W_KV    [d][d] `dtype`       W_K^(-1)·W_V, prepared offline by the caller
 *   dtype   SLIM_BF16 or SLIM_F32
 *   B, d, H B >= 1, H >= 1, d % H == 0
 *   cap     rows per sequence in the cache
 *   variant SLIM_AUTO, SLIM_VARIANT_A or SLIM_VARIANT_B
 *   t_hint  host-side estimate of the attended length, used only by
 *           SLIM_AUTO (<= 0 means cap)
 *   out     float[B][d]          (device, written) concatenated head outputs;
 *           zero for a sequence that was skipped or has nothing to attend to
 *   workspace, ws_bytes  device scratch, >= slim_decode_workspace_bytes(...)
 *   dev_status  device int32 (SLIM_DEV_* bits)
 */
int slim_decode_step(const float* q, const void* k_new, void* Kcache, int32_t* lens, const void* W_KV, int dtype,
                     int B, int d, int H, int64_t cap, int variant, int64_t t_hint, float* out, void* workspace,
                     size_t ws_bytes, int32_t* dev_status, void* stream);

/*
 * slim_decode_step_host — slim_decode_step with the per-step inputs and the
 * output in HOST memory: copies q_host (float[B][d]) and k_new_host ([B][d]
 * `dtype`, or NULL) to device staging space inside `workspace`, runs the
 * step and copies the result back to out_host (float[B][d]), all on
 * `stream`. Host buffers should be page-locked for the copies to be
 * asynchronous. Returns after enqueueing; synchronise `stream` before
 * reading out_host. The cache, lens, W_KV and dev_status stay on the device.
 */
int slim_decode_step_host(const float* q_host, const void* k_new_host, void* Kcache, int32_t* lens,
                          const void* W_KV, int dtype, int B, int d, int H, int64_t cap, int variant, int64_t t_hint,
                          float* out_host, void* workspace, size_t ws_bytes, int32_t* dev_status, void* stream);

/*
 * slim_project_qk — the step's front end: q = x·W_Q and, for self-attention,
 * k = x·W_K for the B input rows of one generation step. Source: section
 * "K-Cache is All You Need", generation phase (the step computes the query of
 * the new token, scores it against the cached K, and appends the new token's
 * key k to the cache; row vectors, as in K = X·W_K).
 *
 *   x       [B][d] in `dtype`      this step's input rows (device, read)
 *   W_Q     [d][d] in `dtype`      (device, read)
 *   W_K     [d][d] in `dtype`, or NULL: q only (a cross-attention step)
 *   dtype   SLIM_BF16: tcgen05 tensor cores where d % 128 == 0 (fp32
 *           accumulation in an order the hardware fixes; k rounded once to
 *           bf16, round-to-nearest-even), CUDA cores otherwise;
 *           SLIM_F32: one fp32 accumulator per output, reduction index
 *           ascending, one fused multiply-add per step (bitwise reproducible)
 *   q_out   float[B][d]            (device, written)
 *   k_out   [B][d] in `dtype`      (device, written); NULL exactly when W_K is
 *   dev_status  device int32 (SLIM_DEV_TIMEOUT only)
 * All pointers 16-byte aligned; SLIM_BF16 needs d % 8 == 0, SLIM_F32 d % 4 == 0.
 */
int slim_project_qk(const void* x, const void* W_Q, const void* W_K, int dtype, int B, int d, float* q_out,
                    void* k_out, int32_t* dev_status, void* stream);

/*
 * slim_decode_step_x — slim_decode_step that starts from the step's input
 * rows: the front end above computes q = x·W_Q and (W_K != NULL) k = x·W_K
 * into the workspace, and the step then attends exactly as slim_decode_step
 * does with those q and k_new (W_K == NULL: cross-attention, no append). Its
 * result equals, bit for bit, slim_project_qk followed by slim_decode_step on
 * the same arguments. The workspace must hold
 * slim_decode_step_x_workspace_bytes(...) bytes (the step's scratch plus q and
 * k); other arguments as for slim_decode_step and slim_project_qk.
 */
size_t slim_decode_step_x_workspace_bytes(int dtype, int B, int d, int H, int64_t cap, int variant);
int slim_decode_step_x(const void* x, const void* W_Q, const void* W_K, void* Kcache, int32_t* lens,
                       const void* W_KV, int dtype, int B, int d, int H, int64_t cap, int variant, int64_t t_hint,
                       float* out, void* workspace, size_t ws_bytes, int32_t* dev_status, void* stream);

/*
 * slim_decode_step_noalloc — slim_decode_step without a caller workspace, for
 * callers that cannot allocate device memory: a plug-in whose host runtime
 * owns all device memory under a plan fixed at start-up and passes it only
 * the tensors it computes on, or a latency-critical decode loop that cannot
 * afford cudaMalloc's implicit device synchronisation. The paper has no
 * counterpart: it is a packaging of the same step. Arguments and results are
 * those of slim_decode_step minus `workspace`/`ws_bytes`; the caller still
 * passes every input and output. This call allocates nothing (no cudaMalloc,
 * no cudaFree, no allocating library routine).
 *
 * Scratch: a buffer of SLIM_NOALLOC_SCRATCH_BYTES compiled into the library,
 * held on every GPU that loads the library until the process exits. Sizes
 * whose slim_decode_workspace_bytes(...) exceeds it are rejected with
 * SLIM_EWORKSPACE before anything is enqueued. The first call on a device
 * looks up the buffer's device address (cudaGetSymbolAddress, with that
 * device current) and remembers it; make that first call before any stream
 * capture. Every call on a device shares the one buffer, which keeps the
 * previous call's contents: the step reads no scratch value it has not
 * written in the same call, so nothing needs clearing, but calls that overlap
 * on the GPU (e.g. on two streams) race with each other and must be
 * serialised by the caller.
 */
#define SLIM_NOALLOC_SCRATCH_BYTES (32 * 1024 * 1024)
/* The size of that buffer as compiled into this library (SLIM_NOALLOC_SCRATCH_BYTES of the header it
 * was built with); host-only, needs no device. */
size_t slim_noalloc_scratch_bytes(void);
int slim_decode_step_noalloc(const float* q, const void* k_new, void* Kcache, int32_t* lens, const void* W_KV,
                             int dtype, int B, int d, int H, int64_t cap, int variant, int64_t t_hint, float* out,
                             int32_t* dev_status, void* stream);

/*
 * slim_prefill_attention — prompt phase: the attention output of the n prompt
 * tokens of every sequence, over the K-only cache. Source: section "K-Cache is
 * All You Need", prompt phase (queries and keys of all prompt tokens in
 * parallel, only K cached, values from K through W_KV). Call it after
 * slim_prefill_k has appended the prompt's keys: the queries are those of the
 * last n cached rows, query j of sequence b at position p = lens[b] - n + j,
 * and it attends causally over rows 0..p (its own key included):
 *     out[b][j][h-cols] = softmax(q_h·K_h[0..p]^T/sqrt(d_h)) · V_h[0..p],
 * V = K·W_KV, computed once for the cached rows into the workspace (ordering
 * (a): every query reuses it), then flash-attention over Q, K and V.
 *
 *   Q        [B][n][d] bf16            the prompt's queries (device, read)
 *   Kcache   [B][cap][d] bf16          (device, read)
 *   lens     int32[B]                  (device, read; not changed)
 *   W_KV     [d][d] bf16
 *   dtype    SLIM_BF16 only; d % 256 == 0, d_h = d/H of 64 or 128
 *   out      float[B][n][d]            (device, written)
 *   workspace >= slim_prefill_attention_workspace_bytes(...), 256-byte aligned
 *   dev_status  SLIM_DEV_BADLEN if lens[b] < n or lens[b] > cap (sequence skipped)
 */
size_t slim_prefill_attention_workspace_bytes(int dtype, int B, int d, int H, int64_t cap);
int slim_prefill_attention(const void* Q, const void* Kcache, const int32_t* lens, const void* W_KV, int dtype,
                           int B, int n, int d, int H, int64_t cap, float* out, void* workspace, size_t ws_bytes,
                           int32_t* dev_status, void* stream);

/*
 * slim_mha_decode_step — the standard multi-head attention generation step
 * over explicit K and V caches, the step Slim attention rewrites: for every
 * sequence b and head h, o[b, h-cols] = softmax(q_h·K_h^T/sqrt(d_h))·V_h.
 * Source: section "K-Cache is All You Need" (standard MHA caches k and v of
 * every token; the article and the paper's abstract compare the K-only step
 * with it: half the context memory, up to 2x faster when the step is
 * memory-bandwidth-bound). Provided as the measured baseline of that claim.
 *
 *   q              float[B][d]          (device, read)
 *   k_new, v_new   [B][d] bf16          this step's key and value, appended at
 *                  row lens[b] of both caches before attending; both NULL =
 *                  no append (attend over lens[b] rows, lens unchanged)
 *   Kcache, Vcache [B][cap][d] bf16     (device; row lens[b] written when appending)
 *   lens           int32[B]             (device; += 1 per appended sequence)
 *   dtype          SLIM_BF16 only (SLIM_F32 returns SLIM_EUNSUPPORTED)
 *   B, d, H        d % 256 == 0, d_h = d/H of 64 or 128
 *   out            float[B][d]          (device, written); zero for a skipped sequence
 *   workspace      >= slim_mha_decode_workspace_bytes(...), 256-byte aligned
 *   dev_status     device int32 (SLIM_DEV_* bits, as for slim_decode_step)
 */
size_t slim_mha_decode_workspace_bytes(int dtype, int B, int d, int H, int64_t cap);
int slim_mha_decode_step(const float* q, const void* k_new, const void* v_new, void* Kcache, void* Vcache,
                         int32_t* lens, int dtype, int B, int d, int H, int64_t cap, float* out, void* workspace,
                         size_t ws_bytes, int32_t* dev_status, void* stream);

/*
 * slim_tune — fills the SLIM_AUTO table for (dtype, B, d, H) by timing both
 * orderings, without append, at each attended length Ts[i] (1 <= Ts[i] <= cap)
 * with CUDA events on `stream`, `reps` repetitions each. It overwrites
 * lens[] with Ts[i] for the measurement and restores it to lens_restore_host
 * (host int32[B]) at the end. Synchronous. Other arguments as in
 * slim_decode_step; Kcache rows 0..max(Ts)-1 must hold finite values.
 */
int slim_tune(const float* q, void* Kcache, int32_t* lens, const int32_t* lens_restore_host, const void* W_KV,
              int dtype, int B, int d, int H, int64_t cap, const int64_t* Ts, int nT, int reps, float* out,
              void* workspace, size_t ws_bytes, int32_t* dev_status, void* stream);

/* slim_tune_record — adds one measured point (milliseconds per step for (a)
 * and (b)) to the SLIM_AUTO table; used by slim_tune and by callers that
 * measured elsewhere. */
int slim_tune_record(int dtype, int B, int d, int H, int64_t T, float ms_a, float ms_b);

/* slim_select_variant — the ordering SLIM_AUTO would run for attended length
 * T: the faster one at the nearest measured T (log scale); ties and an empty
 * table give SLIM_VARIANT_B. */
int slim_select_variant(int dtype, int B, int d, int H, int64_t T);

/* slim_tune_clear — empties the SLIM_AUTO table. */
void slim_tune_clear(void);

/* slim_strerror — static description of a return code or SLIM_DEV_* bit set. */
const char* slim_strerror(int code);

/* slim_last_launch_count — number of kernels the last successful call on this
 * host thread enqueued. */
int slim_last_launch_count(void);

/* slim_timing_enable — measurement aid. With n > 0, every following
 * slim_decode_step on this host thread records a pair of CUDA events
 * (owned by the library, timing enabled) on `stream` immediately before and
 * after its split kernel (the kernel that streams the K cache), cycling
 * through n pairs; this also works inside CUDA-graph capture, where the
 * records become event nodes. n = 0 destroys the events. Returns SLIM_OK,
 * SLIM_EINVAL (n < 0) or SLIM_ECUDA. Host-side only; allocates no device memory. */
int slim_timing_enable(int n);

/* slim_timing_read — after `stream` has been synchronised, writes the
 * elapsed milliseconds of pair i into ms[i] for i < min(n, pairs recorded)
 * and returns that count (negative SLIM_E* on error). */
int slim_timing_read(float* ms, int n);

/*
 * slim_debug_stall_next — test hook for the failure path. The next
 * slim_decode_step on this host thread that runs the tcgen05 split kernel
 * (ordering (b), bf16 cache) makes that kernel's MMA warp wait on a barrier
 * that nothing completes, with every wait of that kernel limited to wait_ns
 * nanoseconds (1000 <= wait_ns <= 1e9) instead of the usual second. The
 * kernel then ORs SLIM_DEV_TIMEOUT into *dev_status, lets every copy it
 * issued land, frees its tensor memory and returns; that step's output and
 * the lengths it advances are not meaningful, the cache is not corrupted and
 * the context stays usable. Returns SLIM_OK, or SLIM_EINVAL for wait_ns out
 * of range. Host-side only.
 */
int slim_debug_stall_next(int64_t wait_ns);

/* slim_version — ABI version (major*100 + minor). */
int slim_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SLIM_H_ */
