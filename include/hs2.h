/*
 * hs2.h -- C ABI of libhs2, the decode step of a HySparse2 Cross-Decoder hybrid
 * block on NVIDIA B200 (sm_100a).
 *
 * The step (sources: web coverage of the HySparse2 architecture paper):
 *   1. a full-attention layer with one shared K/V head and h_q query heads (MQA)
 *      attends over the whole context and scores every key
 *      (toolnavs article 2080, fr "Ce que fait HySparse2", KV Reuse paragraph;
 *       "Les chiffres mesurés" for MQA);
 *   2. token-level selection keeps the most recent `window` (128) positions and
 *      the top `k_sel` (1024) positions outside that window
 *      (same article, fr/ko, paragraph on selection granularity; "Luo Fuli Teases
 *       Xiaomi MiMo-V3 Architecture: HySparse2 Enables Early Prefill Exit",
 *       paragraph on token granularity);
 *   3. each following sparse-attention layer, with its own queries, attends only
 *      to those positions of the same KV cache (same article, KV Reuse paragraph).
 * Around the step: hs2_kv_append writes the new tokens' K and V rows before it (E4M3
 * with a per-token scale for an FP8 cache); hs2_prefill_attn runs the full layer over
 * a chunk of new tokens (chunked prefill, no selection); hs2_full_attn_select_blocks
 * keeps whole 64-token blocks instead of tokens (the first-generation scheme the
 * pages compare against).
 * The pages give no importance formula.  This library takes a key's importance as
 * max over query heads h of exp(s_hj - lse_h), the full layer's softmax
 * probability, with ties going to the lower position.
 *
 * Conventions shared by every call
 *   - Pointers named "device" point to device memory of the current CUDA device.
 *     The caller owns all memory; the library allocates nothing and keeps no
 *     pointer after a call returns.
 *   - Every compute call is asynchronous on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream) and enqueues only kernels and memsets, so it can be
 *     captured in a CUDA graph.
 *   - Host-side validation failures return an error before anything is enqueued.
 *     Launch failures return HS2_ERR_CUDA.  Errors found by the kernels (a bad
 *     length, an index out of range) are recorded in the workspace's status word
 *     and read with hs2_check_device_status().
 *   - head_dim must be 128.  h_q must be a multiple of 16 in [16, 128].
 *     n_q (query tokens per sequence) is in [1, 64] (hs2_prefill_attn: [1, 65536]);
 *     batch * n_q <= 65535 (hs2_prefill_attn: batch * ceil(n_q * h_q / 128) <= 65535).
 *     window >= 1, k_sel >= 1,
 *     window + k_sel <= 4096.  Otherwise HS2_ERR_UNSUPPORTED.
 *   - Query token i of sequence b sits at position p = lens[b] - n_q + i and sees
 *     keys [0, p]; 1 <= n_q <= lens[b] <= max_len is required (checked on the
 *     device: a violating sequence sets HS2_ERR_BAD_LENGTH and is clamped).
 *   - All of q, k, v, out and the workspace must be 16-byte aligned; rows are
 *     dense (strides are implied by the shapes given below).
 */
#ifndef HS2_H_
#define HS2_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define HS2_API __attribute__((visibility("default")))
#else
#define HS2_API
#endif

typedef struct CUstream_st* hs2_stream_t; /* identical to cudaStream_t */

typedef enum hs2_status {
  HS2_OK = 0,
  HS2_ERR_INVALID_ARGUMENT = 1,    /* null pointer, bad size, misalignment        */
  HS2_ERR_UNSUPPORTED = 2,         /* outside the supported ranges listed above    */
  HS2_ERR_WORKSPACE_TOO_SMALL = 3, /* ws_bytes < hs2_workspace_bytes(...)          */
  HS2_ERR_CUDA = 4,                /* a CUDA runtime call failed                   */
  HS2_ERR_DEVICE_TIMEOUT = 5,      /* a bounded device-side wait gave up           */
  HS2_ERR_INDEX_OUT_OF_RANGE = 6,  /* sparse index outside [0, lens[b]) and != -1  */
  HS2_ERR_BAD_LENGTH = 7           /* lens[b] outside [n_q, max_len]               */
} hs2_status;

typedef enum hs2_kv_dtype {
  HS2_KV_BF16 = 0,     /* K and V are bfloat16                                      */
  HS2_KV_FP8_E4M3 = 1  /* K and V are OCP FP8 E4M3 ("fn") codes with per-token
                          float32 scales: value = decode(code) * scale[b][j]        */
} hs2_kv_dtype;

/* The shared KV cache of one hybrid block (one K/V head: MQA).
 *   k, v     device, [batch][max_len][head_dim], head_dim contiguous; element type
 *            per `dtype` (2 bytes bf16 or 1 byte E4M3 code).  Only rows [0, lens[b])
 *            are read; the rest may hold anything, NaN included.
 *   k_scale, v_scale  device float32 [batch][max_len]; required for FP8, must be
 *            NULL for bf16.
 *   lens     device int32 [batch].                                                */
typedef struct hs2_kv {
  const void* k;
  const void* v;
  const float* k_scale;
  const float* v_scale;
  const int32_t* lens;
  int32_t batch;
  int32_t max_len;
  int32_t head_dim;
  int32_t dtype; /* hs2_kv_dtype */
} hs2_kv;

/* Bytes of workspace that the calls below need for these sizes (0 if the sizes are
 * unsupported).  One workspace serves hs2_full_attn_select and every following
 * hs2_sparse_attn of the same step.  It must be zero-filled once before first use;
 * afterwards the library keeps it consistent itself.  Calls sharing a workspace
 * must be ordered (same stream, or otherwise serialised). */
HS2_API size_t hs2_workspace_bytes(int batch, int n_q, int h_q, int max_len, int window,
                           int k_sel, int dtype);

/* Byte offset, within a workspace of these sizes, of the float64 log-sum-exp that the
 * full layer leaves there: double [batch][n_q][h_q], natural log, the values the token
 * selection shifts the heads' scores by.  Valid after hs2_full_attn or
 * hs2_full_attn_select until the next call that uses the workspace.  (size_t)-1 if the
 * sizes are unsupported.  A diagnostic: the `lse` output of those calls is the same
 * value rounded to float32. */
HS2_API size_t hs2_workspace_lse64_offset(int batch, int n_q, int h_q, int max_len,
                                          int window, int k_sel, int dtype);

/* Full-attention layer + token selection (steps 1 and 2).
 *   q        device bf16 [batch][n_q][h_q][128].
 *   sm_scale softmax scale applied to q.k (normally 1/sqrt(128) as float32).
 *   out      device float32 [batch][n_q][h_q][128]: softmax(s) @ V over keys [0, p].
 *   idx      device int32 [batch][n_q][window + k_sel]: the ascending union of
 *            [max(0, p-window+1), p] and the top-k_sel positions of [0, p-window]
 *            by (importance desc, position asc); when p+1 <= window + k_sel it is
 *            all of [0, p]; unused slots are -1.
 *   lse      device float32 [batch][n_q][h_q] natural-log sum-exp of the logits,
 *            or NULL.
 * Equivalent to hs2_full_attn followed by hs2_select on the same workspace.  For one new
 * token per sequence on a bf16 cache and for an FP8 cache, with h_q <= 64
 * (hs2_select_fused), it is a single cooperative kernel: the full layer's CTAs merge
 * their split partials and select the tokens in its tail, re-scoring only the keys whose
 * bound u_j = max_h s_hj can reach the top k_sel, so K is read once.  The index set is
 * the same either way outside the tie band (keys whose exact importances differ by less
 * than the lse's rounding); outputs can differ between runs in their last bits unless
 * hs2_set_deterministic is on. */
HS2_API hs2_status hs2_full_attn_select(const void* q, int n_q, int h_q, const hs2_kv* kv,
                                int window, int k_sel, float sm_scale, float* out,
                                int32_t* idx, float* lse, void* workspace,
                                size_t ws_bytes, hs2_stream_t stream);

/* Step 1 alone: split-K flash-decode over every visible key, writing `out` and
 * (if non-NULL) `lse`, and leaving the per-head log-sum-exp in the workspace for
 * hs2_select.  Arguments as above. */
HS2_API hs2_status hs2_full_attn(const void* q, int n_q, int h_q, const hs2_kv* kv,
                         int window, int k_sel, float sm_scale, float* out, float* lse,
                         void* workspace, size_t ws_bytes, hs2_stream_t stream);

/* Step 2 alone: importance of every key outside the window and the exact top-k_sel
 * selection merged with the window, into `idx`.  Must follow hs2_full_attn with the
 * same q, kv, sizes and workspace, on the same stream. */
HS2_API hs2_status hs2_select(const void* q, int n_q, int h_q, const hs2_kv* kv, int window,
                      int k_sel, float sm_scale, int32_t* idx, void* workspace,
                      size_t ws_bytes, hs2_stream_t stream);

/* Block-level selection, the first-generation scheme that the pages set token-level
 * selection against ("Luo Fuli Teases Xiaomi MiMo-V3 Architecture ...", paragraphs on
 * block selection with 64-token blocks and on the ablation at the same attention
 * budget): a comparator, not the method's own step.
 *   block    positions per block (the pages' blocks hold 64), >= 2; k_sel must be a
 *            multiple of block and k_sel / block <= 1024.
 *   idx      device int32 [batch][n_q][window + k_sel]: positions [0, p-window] form
 *            aligned blocks [c*block, (c+1)*block), the last one cut at p-window; a
 *            block scores the largest importance among its positions (a reading: the
 *            pages give no block score); the k_sel / block best blocks, ties to the
 *            lower block, are kept whole, in ascending order, then the window
 *            [p-window+1, p], then -1.  With no more blocks than k_sel / block, all of
 *            [0, p].
 * Other arguments, workspace and ordering as hs2_full_attn_select / hs2_select.
 * HS2_ERR_UNSUPPORTED for a block size outside these limits, or when the row's
 * ceil(max_len / block) block keys do not fit the kernel's shared memory (about
 * 40000 blocks at 16 heads). */
HS2_API hs2_status hs2_full_attn_select_blocks(const void* q, int n_q, int h_q,
                                               const hs2_kv* kv, int window, int k_sel,
                                               int block, float sm_scale, float* out,
                                               int32_t* idx, float* lse, void* workspace,
                                               size_t ws_bytes, hs2_stream_t stream);

/* Block-level selection alone; must follow hs2_full_attn with the same q, kv, sizes
 * and workspace, on the same stream. */
HS2_API hs2_status hs2_select_blocks(const void* q, int n_q, int h_q, const hs2_kv* kv,
                                     int window, int k_sel, int block, float sm_scale,
                                     int32_t* idx, void* workspace, size_t ws_bytes,
                                     hs2_stream_t stream);

/* Chunked prefill of the Cross-Decoder's full layer: the full-attention layer for a
 * chunk of n_q new tokens per sequence (already appended to the cache), the same
 * attention as hs2_full_attn (token i at p = lens[b] - n_q + i sees keys [0, p]), with
 * no selection ("Luo Fuli Teases Xiaomi MiMo-V3 Architecture ..." and toolnavs
 * article 2080: the full layers attend over the whole context).  Tensor cores: 128
 * query rows (128 / h_q tokens x h_q heads) share each K/V tile.
 *   q        device bf16 [batch][n_q][h_q][128];  n_q in [1, 65536], n_q <= max_len.
 *   h_q      16, 32, 48, 64 or 128.  kv: bf16 caches only (else HS2_ERR_UNSUPPORTED).
 *   out      device float32 [batch][n_q][h_q][128]; lse float32 [batch][n_q][h_q] or NULL.
 *   workspace  at least hs2_prefill_workspace_bytes(batch, n_q, h_q, max_len, dtype)
 *            bytes (split partials; zero-filled once, as for the decode calls).
 * A sequence with lens[b] < n_q reports HS2_ERR_BAD_LENGTH through the workspace's
 * status word (hs2_check_device_status). */
HS2_API size_t hs2_prefill_workspace_bytes(int batch, int n_q, int h_q, int max_len,
                                           int dtype);
HS2_API hs2_status hs2_prefill_attn(const void* q, int n_q, int h_q, const hs2_kv* kv,
                                    float sm_scale, float* out, float* lse, void* workspace,
                                    size_t ws_bytes, hs2_stream_t stream);

/* One reusing sparse-attention layer (step 3).
 *   q_layer   device bf16 [batch][n_q][h_q][128], this layer's queries.
 *   idx       device int32 [batch][n_q][idx_width]: positions to attend to (any
 *             order, duplicates counted as given); -1 entries are skipped.  An entry
 *             outside [0, lens[b]) is skipped and sets HS2_ERR_INDEX_OUT_OF_RANGE.
 *   out       device float32 [batch][n_q][h_q][128]; a row whose set is empty gets 0.
 * idx_width in [1, 4096]; the workspace must come from hs2_workspace_bytes with
 * window + k_sel >= idx_width.
 * Overlap: the layer's kernel may start while the previous kernel on the stream is
 * still finishing when that kernel is this library's (programmatic dependent launch);
 * it reads q_layer, idx and the cache right away and waits for that kernel to end only
 * before writing `out`.  The library calls that write those inputs (hs2_select and
 * hs2_full_attn_select the index set, hs2_kv_append the cache rows and lengths) finish
 * those writes before they let the next kernel start.
 * After any other kernel (not this library's) the layer starts when it has ended. */
HS2_API hs2_status hs2_sparse_attn(const void* q_layer, int n_q, int h_q, const hs2_kv* kv,
                           const int32_t* idx, int idx_width, float sm_scale, float* out,
                           void* workspace, size_t ws_bytes, hs2_stream_t stream);

/* One reusing sparse-attention layer for callers that cannot allocate device memory
 * (no counterpart in the paper; a deployment aid).  It computes the same layer as
 * hs2_sparse_attn, within the same tolerances (for h_q <= 64 with a different kernel:
 * CUDA-core gathers and a separate split merge), with the same arguments except the
 * workspace: its scratch
 * (the split partials) lives in a fixed 4 MiB array inside the library,
 * which every GPU that loads the library keeps until the process exits.  Callers that
 * hand out all device memory from their own pool, or that must not call cudaMalloc
 * mid-step (it can synchronise the device), use this entry point.
 *   device_status  device uint32 into which the kernels OR (1 << code) for each
 *                  device-side error (HS2_ERR_INDEX_OUT_OF_RANGE: an index outside
 *                  [-1, lens[b]); lengths outside [n_q, max_len] are clamped without a
 *                  report).  The caller clears it.  May be NULL: the errors then
 *                  accumulate in a word of the library's array that nothing reads or
 *                  clears.
 * Limit: 256 + B*n_q*ceil(idx_width/64)*h_q*520 bytes (two regions, each rounded up to
 * 256) must fit in 4 MiB, e.g. B*n_q*h_q <= 448 at idx_width 1152;
 * larger sizes return HS2_ERR_WORKSPACE_TOO_SMALL before anything is enqueued.
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress)
 * and should come before any stream capture on that device.  All calls on a device
 * share the array: calls whose kernels may overlap on the GPU race and must be
 * serialised (same stream, or events between them). */
HS2_API hs2_status hs2_sparse_attn_noalloc(const void* q_layer, int n_q, int h_q,
                                           const hs2_kv* kv, const int32_t* idx,
                                           int idx_width, float sm_scale, float* out,
                                           uint32_t* device_status, hs2_stream_t stream);

/* Appends n_new tokens to every sequence of the cache: the step before the full layer in
 * a decode loop.  (The pages say only that the KV cache may be FP8; per-token
 * absolute-maximum scaling of the new rows is this library's reading.)
 *   k_new, v_new  device bf16 [batch][n_new][128]: the new tokens' keys and values.
 *   kv            the cache.  Rows lens[b] .. lens[b] + n_new - 1 of K and V (and, for
 *                 FP8, of k_scale / v_scale) are written: the arrays behind kv change.
 *   lens          device int32 [batch], the cache's lengths (the array kv->lens points
 *                 to): read, then grown by n_new.
 * FP8: each new row becomes E4M3 codes with its own float32 scale s = amax|row| / 448 and
 * code = row / s rounded to nearest even, saturating at 448 (both divisions IEEE
 * float32); an all-zero row gets s = 1.  bf16: the rows are copied.
 * A sequence with lens[b] + n_new > max_len is left unchanged and sets
 * HS2_ERR_BAD_LENGTH in the workspace's status word.  n_new in [1, 64]; k_new and v_new
 * 16-byte aligned.  Like the other calls it may start while an earlier kernel of this
 * library is finishing, but it waits for that kernel before reading or writing. */
HS2_API hs2_status hs2_kv_append(const void* k_new, const void* v_new, int n_new,
                                 const hs2_kv* kv, int32_t* lens, void* workspace,
                                 size_t ws_bytes, hs2_stream_t stream);

/* Synchronises `stream` and returns an error the kernels recorded since the last check
 * (HS2_OK if none), then clears them all.  Each kind of error sets its own bit of the
 * workspace's status word, so when several kinds were recorded the call returns the
 * lowest-numbered code among them (the order of hs2_status, not the order in time).
 * After HS2_ERR_DEVICE_TIMEOUT the workspace's contents are undefined: zero-fill it again
 * before the next call that uses it. */
HS2_API hs2_status hs2_check_device_status(void* workspace, hs2_stream_t stream);

/* Reproducibility switch (process-wide; 0 by default).  By default the one-launch full
 * layer shares each row's key tiles out among its CTAs at run time (CTAs slowed by the
 * memory system take fewer tiles), so the grouping of the float32 partial sums, and with
 * it the last bits of the outputs and of the lse, can differ between two runs on the same
 * inputs; the index set differs only where two keys' exact scores are within the lse's
 * rounding (~1e-7).  With `on` nonzero every CTA takes a fixed chunk of keys and repeated
 * runs are bitwise identical, at some cost in speed (on a B200 about 3 % of the step at
 * 8 x 131072 bf16 keys and 6 % at 1M FP8 keys, where the memory system's uneven pace across
 * SMs is no longer evened out).  Applies to the launches that follow; not synchronised
 * between host threads. */
HS2_API void hs2_set_deterministic(int on);

/* Test hook for the error path of the bounded device-side waits; not for production.
 *   mode 1: the bf16 one-token full-layer kernel issues no loads and no MMAs, so its
 *           softmax warps' first wait on an MMA result runs out (after about 10 us);
 *   mode 2: the fused selection tail's row barriers wait for one CTA more than the row
 *           has, so each runs out (after about 10 us);
 *   mode 0: normal operation (the default).
 * A wait that runs out records HS2_ERR_DEVICE_TIMEOUT and the kernel finishes with no
 * copy or MMA of its own in flight; outputs are then undefined and the workspace must be
 * zero-filled again before its next use.  The setting is process-wide, applies to the
 * launches that follow, and is not synchronised between host threads. */
HS2_API void hs2_debug_stall_waits(int mode);

/* Static description of a status code (never NULL). */
HS2_API const char* hs2_status_string(hs2_status status);

/* 1 if hs2_full_attn_select runs as a single kernel for these sizes (the one-token
 * tensor-core full layer, which merges its split partials and selects the tokens in its
 * own tail), 0 if it runs as the full layer, the split merge and separate selection
 * kernels.  The results are the same either way; only the launches differ. */
HS2_API int hs2_select_fused(int n_q, int h_q, int dtype);

/* Text of the last CUDA error seen by this thread's calls ("" if none). */
HS2_API const char* hs2_last_cuda_error(void);

/* ABI version of this header; bumped on any incompatible change. */
HS2_API int hs2_abi_version(void);

#define HS2_ABI_VERSION 1

#ifdef __cplusplus
}
#endif

#endif /* HS2_H_ */
