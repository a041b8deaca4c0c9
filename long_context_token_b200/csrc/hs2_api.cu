// Host side of the libhs2 C ABI: argument validation, workspace layout and the
// launch sequence of each call.  Nothing here allocates device memory.
#include <stdio.h>
#include <string.h>

#include "hs2_internal.cuh"
#include "tc_common.cuh"

namespace hs2 {

static thread_local char g_last_cuda_error[256] = "";

static hs2_status cuda_fail(cudaError_t e, const char* what) {
  snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", what,
           cudaGetErrorString(e));
  return HS2_ERR_CUDA;
}

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Target of ~4 CTAs per SM of a 148-SM B200 for the key-chunk kernels; fixed so
// that the workspace layout does not depend on the device it runs on.
constexpr int kTargetCtas = 4 * 148;
constexpr int kMinChunk = 256;
constexpr int kChunk4 = 64;

// The bounded-wait test hook (hs2_debug_stall_waits): copied into every full-layer launch.
static int g_stall_test = 0;
// hs2_set_deterministic: static key chunks in the full layer (no run-time tile sharing).
static int g_deterministic = 0;

// `row_ctas`: CTAs of one key chunk across the batch (one per (sequence, token) row,
// or per group of G tokens in the several-token kernel).
int plan_splits1(int row_ctas, int max_len, int /*num_sms*/) {
  int splits = (kTargetCtas + row_ctas - 1) / row_ctas;
  const int max_splits = (max_len + kMinChunk - 1) / kMinChunk;
  if (splits > max_splits) splits = max_splits;
  if (splits < 1) splits = 1;
  return splits;
}

static int chunk_for(int max_len, int splits) {
  int chunk = (max_len + splits - 1) / splits;
  return (chunk + 31) / 32 * 32;
}

int plan_splits4(int idx_width) { return (idx_width + kChunk4 - 1) / kChunk4; }

bool make_layout(int batch, int n_q, int h, int max_len, int window, int k_sel, int dtype,
                 WsLayout* L) {
  WsLayout w;
  w.bq = batch * n_q;
  w.h = h;
  w.max_len = max_len;
  w.window = window;
  w.k_sel = k_sel;
  const int row_ctas = dtype == HS2_KV_BF16 && mq_eligible(n_q, h)
                           ? batch * ((n_q + mq_tokens_per_cta(h) - 1) / mq_tokens_per_cta(h))
                           : w.bq;
  w.splits1 = plan_splits1(row_ctas, max_len, kSmCountBound);
  w.splits4 = plan_splits4(kMaxIdxWidth);  // capacity for any idx_width
  const size_t bq = (size_t)w.bq, ml = (size_t)max_len, hh = (size_t)h;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, 256);
    return at;
  };
  // Regions that depend only on (bq, h): status and the sparse-layer state.
  w.status = take(sizeof(uint32_t));
  w.part4_o = take(bq * w.splits4 * hh * kHeadDim * sizeof(float));
  w.part4_ml = take(bq * w.splits4 * hh * 2 * sizeof(float));
  // Regions of the full layer and the selection.
  w.clear_begin = off;
  w.hist = take(bq * kHistBins * sizeof(uint32_t));
  w.rowmax = take(bq * kMaxHeads * sizeof(uint32_t));
  w.counters = take(bq * 8 * sizeof(uint32_t));
  w.clear_end = off;
  w.selmeta = take(bq * 4 * sizeof(uint32_t));
  w.part1_o = take(bq * w.splits1 * hh * kHeadDim * sizeof(float));
  w.part1_ml = take(bq * w.splits1 * hh * 2 * sizeof(float));
  w.lse64 = take(bq * hh * sizeof(double));
  w.tbuf = take(bq * ml * sizeof(float));
  w.use_sbuf = sbuf_eligible(n_q, h, dtype);
  w.sbuf = take(w.use_sbuf ? bq * ml * hh * sizeof(float) : 0);
  w.direct = take(bq * (size_t)k_sel * sizeof(int32_t));
  // (rows of ld_u entries for the fused tail, whose 16-byte copies need aligned rows)
  const size_t ld_u = (ml + 31) / 32 * 32;
  w.cand_t = take(bq * ld_u * sizeof(float));
  w.cand_j = take(bq * ld_u * sizeof(int32_t));
  w.band_t = take(bq * ml * sizeof(double));
  w.band_j = take(bq * ml * sizeof(int32_t));
  w.ld_u = (max_len + 31) / 32 * 32;
  w.ubuf = take(bq * (size_t)w.ld_u * sizeof(float));
  w.rowcnt = take(bq * (size_t)kSmCountBound * sizeof(uint32_t));
  w.total = off;
  *L = w;
  return true;
}

// Bytes of the leading part of the workspace that a sparse layer uses.
static size_t sparse_prefix_bytes(const WsLayout& w) { return w.clear_begin; }

static bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

constexpr long long kMaxGridY = 65535;

static hs2_status check_shape(int batch, int n_q, int h, int max_len, int window, int k_sel) {
  if (batch < 1 || max_len < 1) return HS2_ERR_INVALID_ARGUMENT;
  if (n_q < 1 || n_q > kMaxNq) return HS2_ERR_UNSUPPORTED;
  if (h < 16 || h > kMaxHeads || (h % 16) != 0) return HS2_ERR_UNSUPPORTED;
  if (window < 1 || k_sel < 1 || window + k_sel > kMaxIdxWidth) return HS2_ERR_UNSUPPORTED;
  if (max_len < n_q) return HS2_ERR_INVALID_ARGUMENT;
  if ((long long)batch * (long long)max_len >= (1ll << 31)) return HS2_ERR_UNSUPPORTED;
  // One grid row per (sequence, token): the grid's y extent.
  if ((long long)batch * n_q > kMaxGridY) return HS2_ERR_UNSUPPORTED;
  return HS2_OK;
}

static hs2_status check_kv(const hs2_kv* kv) {
  if (!kv || !kv->k || !kv->v || !kv->lens) return HS2_ERR_INVALID_ARGUMENT;
  if (kv->head_dim != kHeadDim) return HS2_ERR_UNSUPPORTED;
  if (kv->dtype == HS2_KV_BF16) {
    if (kv->k_scale || kv->v_scale) return HS2_ERR_INVALID_ARGUMENT;
  } else if (kv->dtype == HS2_KV_FP8_E4M3) {
    if (!kv->k_scale || !kv->v_scale) return HS2_ERR_INVALID_ARGUMENT;
  } else {
    return HS2_ERR_UNSUPPORTED;
  }
  if (!aligned16(kv->k) || !aligned16(kv->v)) return HS2_ERR_INVALID_ARGUMENT;
  return HS2_OK;
}

static KvView view_of(const hs2_kv* kv) {
  KvView v;
  v.k = kv->k;
  v.v = kv->v;
  v.k_scale = kv->k_scale;
  v.v_scale = kv->v_scale;
  v.lens = kv->lens;
  v.batch = kv->batch;
  v.max_len = kv->max_len;
  v.fp8 = kv->dtype == HS2_KV_FP8_E4M3;
  return v;
}

struct Prepared {
  WsLayout w;
};

static hs2_status prepare(const void* q, int n_q, int h, const hs2_kv* kv, int window,
                          int k_sel, void* ws, size_t ws_bytes, Prepared* P) {
  hs2_status st = check_kv(kv);
  if (st != HS2_OK) return st;
  st = check_shape(kv->batch, n_q, h, kv->max_len, window, k_sel);
  if (st != HS2_OK) return st;
  if (!q || !ws) return HS2_ERR_INVALID_ARGUMENT;
  if (!aligned16(q) || !aligned16(ws)) return HS2_ERR_INVALID_ARGUMENT;
  make_layout(kv->batch, n_q, h, kv->max_len, window, k_sel, kv->dtype, &P->w);
  if (ws_bytes < P->w.total) return HS2_ERR_WORKSPACE_TOO_SMALL;
  return HS2_OK;
}

// Key chunks of the one-token tensor-core full layer (bf16 or FP8): about one CTA per SM,
// chunks of whole 128-key tiles, at most the workspace's split count.
static void plan_decode_splits(const hs2_kv* kv, int n_q, const WsLayout& w, int* splits_out,
                               int* chunk_out) {
  const int bq = kv->batch * n_q;
  int splits = device_sm_count() / bq;
  if (splits > w.splits1) splits = w.splits1;
  if (splits > kSmCountBound) splits = kSmCountBound;  // the fused tail's per-row bound
  if (splits < 1) splits = 1;
  int chunk = (kv->max_len + splits - 1) / splits;
  chunk = (chunk + 127) / 128 * 128;
  *splits_out = (kv->max_len + chunk - 1) / chunk;
  *chunk_out = chunk;
}

// Shapes whose full layer runs on the one-token tensor-core kernels, which merge their
// split partials themselves and can select the row's tokens in the same launch.
static bool fused_full_layer(const hs2_kv* kv, int n_q, int h) {
  if (kv->dtype == HS2_KV_BF16) return h <= 64 && !mq_eligible(n_q, h);
  return h <= 64;  // FP8: the E4M3 tensor-core kernel for any number of tokens
}

// The full layer.  On the fused shapes (fused_full_layer) the kernel merges its split
// partials itself and, with `idx` non-null, also writes the token selection (then
// run_select must not follow); elsewhere the split merge follows as its own kernel.
static hs2_status run_full(const void* q, int n_q, int h, const hs2_kv* kv, int window,
                           int k_sel, float sm_scale, float* out, float* lse, void* ws,
                           const WsLayout& w, cudaStream_t s, int32_t* idx = nullptr) {
  FullParams p;
  p.q = static_cast<const uint16_t*>(q);
  p.kv = view_of(kv);
  p.n_q = n_q;
  p.h = h;
  p.window = window;
  p.k_sel = k_sel;
  p.sm_scale = sm_scale;
  p.splits1 = w.splits1;
  p.chunk1 = chunk_for(kv->max_len, w.splits1);
  p.part_o = ws_ptr<float>(ws, w.part1_o);
  p.part_ml = ws_ptr<float>(ws, w.part1_ml);
  p.status = ws_ptr<uint32_t>(ws, w.status);
  p.stall_test = g_stall_test;
  p.deterministic = g_deterministic;
  if (fused_full_layer(kv, n_q, h)) {
    p.fuse = idx ? 2 : 1;
    p.out = out;
    p.lse_out = lse;
    p.lse64 = ws_ptr<double>(ws, w.lse64);
    p.ubuf = ws_ptr<float>(ws, w.ubuf);
    p.ld_u = w.ld_u;
    p.uhist = ws_ptr<uint32_t>(ws, w.hist);
    p.rowsync = ws_ptr<uint32_t>(ws, w.counters);
    p.rowmax = ws_ptr<uint32_t>(ws, w.rowmax);
    p.cand_t = ws_ptr<float>(ws, w.cand_t);
    p.cand_j = ws_ptr<int32_t>(ws, w.cand_j);
    p.band_t = ws_ptr<double>(ws, w.band_t);
    p.band_j = ws_ptr<int32_t>(ws, w.band_j);
    p.rowcnt = ws_ptr<uint32_t>(ws, w.rowcnt);
    p.sel_idx = idx;
  }
  bool log2_partials = false;
  cudaError_t e;
  if (kv->dtype == HS2_KV_FP8_E4M3 && h <= 64) {
    // Tensor-core flash-decode: the E4M3 tiles go straight into kind::f8f6f4 MMAs.
    CUtensorMap tk, tv;
    const uint64_t rows = (uint64_t)kv->batch * kv->max_len;
    if (!make_tmap_2d(&tk, kv->k, CU_TENSOR_MAP_DATA_TYPE_UINT8, kHeadDim, rows, kHeadDim, 128,
                      128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_2d(&tv, kv->v, CU_TENSOR_MAP_DATA_TYPE_UINT8, kHeadDim, rows, kHeadDim, 128,
                      128, CU_TENSOR_MAP_SWIZZLE_128B))
      return cuda_fail(cudaErrorInvalidValue, "tensor maps of K/V");
    const int bq = kv->batch * n_q;
    plan_decode_splits(kv, n_q, w, &p.splits1, &p.chunk1);
    // The stored logits serve a separate hs2_select call only.
    p.sbuf = w.use_sbuf && p.fuse != 2 ? ws_ptr<float>(ws, w.sbuf) : nullptr;
    e = launch_full_attn_fp8(p, tk, tv, bq, s);
    if (e != cudaSuccess) return cuda_fail(e, "full-attention launch");
    if (p.fuse) return HS2_OK;
    log2_partials = true;
  } else if (kv->dtype == HS2_KV_BF16 && mq_eligible(n_q, h)) {
    // Several new tokens (or 128 heads): 128 query rows of one sequence per CTA, so
    // each K/V tile is read once for G = 128 / h tokens; chunks of 64-key tiles.
    CUtensorMap tk, tv;
    const uint64_t rows = (uint64_t)kv->batch * kv->max_len;
    if (!make_tmap_2d(&tk, kv->k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kHeadDim, rows,
                      kHeadDim * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_2d(&tv, kv->v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kHeadDim, rows,
                      kHeadDim * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B))
      return cuda_fail(cudaErrorInvalidValue, "tensor maps of K/V");
    const int G = mq_tokens_per_cta(h);
    const int ctas_per_split = kv->batch * ((n_q + G - 1) / G);
    int splits = device_sm_count() / ctas_per_split;
    if (splits > w.splits1) splits = w.splits1;
    if (splits < 1) splits = 1;
    int chunk = (kv->max_len + splits - 1) / splits;
    chunk = (chunk + 63) / 64 * 64;
    p.splits1 = (kv->max_len + chunk - 1) / chunk;
    p.chunk1 = chunk;
    e = launch_full_attn_mq(p, tk, tv, kv->batch, s);
    log2_partials = true;
  } else if (kv->dtype == HS2_KV_BF16 && h <= 64) {
    // Tensor-core flash-decode: about one CTA per SM, chunks of whole 128-key tiles.
    CUtensorMap tk, tv;
    const uint64_t rows = (uint64_t)kv->batch * kv->max_len;
    if (!make_tmap_2d(&tk, kv->k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kHeadDim, rows,
                      kHeadDim * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_tmap_2d(&tv, kv->v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kHeadDim, rows,
                      kHeadDim * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
      return cuda_fail(cudaErrorInvalidValue, "tensor maps of K/V");
    const int bq = kv->batch * n_q;
    plan_decode_splits(kv, n_q, w, &p.splits1, &p.chunk1);
    // The stored logits serve a separate hs2_select call only.
    p.sbuf = w.use_sbuf && p.fuse != 2 ? ws_ptr<float>(ws, w.sbuf) : nullptr;
    e = launch_full_attn_tc(p, tk, tv, bq, s);
    if (e != cudaSuccess) return cuda_fail(e, "full-attention launch");
    if (p.fuse) return HS2_OK;
    log2_partials = true;
  } else {
    e = launch_full_attn(p, kv->batch, s);
  }
  if (e != cudaSuccess) return cuda_fail(e, "full-attention launch");
  MergeParams m;
  m.part_o = p.part_o;
  m.part_ml = p.part_ml;
  m.splits = p.splits1;
  m.h = h;
  m.out = out;
  m.lse_out = lse;
  m.lse64 = ws_ptr<double>(ws, w.lse64);
  e = launch_merge(m, kv->batch * n_q, log2_partials, s);
  return e == cudaSuccess ? HS2_OK : cuda_fail(e, "full-attention merge launch");
}

static hs2_status run_select(const void* q, int n_q, int h, const hs2_kv* kv, int window,
                             int k_sel, float sm_scale, int32_t* idx, void* ws,
                             const WsLayout& w, cudaStream_t s, int block = 1) {
  // The histogram and counters start at zero: the workspace is zero-filled before first
  // use and every selection leaves them at zero when it finishes.
  cudaError_t e = cudaSuccess;
  SelectParams p;
  p.q = static_cast<const uint16_t*>(q);
  p.kv = view_of(kv);
  p.n_q = n_q;
  p.h = h;
  p.window = window;
  p.k_sel = k_sel;
  p.sm_scale = sm_scale;
  p.splits2 = w.splits1;
  p.chunk2 = chunk_for(kv->max_len, w.splits1);
  p.chunk3 = kChunk3Keys;
  p.splits3 = (kv->max_len + kChunk3Keys - 1) / kChunk3Keys;
  p.lse64 = ws_ptr<double>(ws, w.lse64);
  p.sbuf = w.use_sbuf ? ws_ptr<float>(ws, w.sbuf) : nullptr;
  p.tbuf = ws_ptr<float>(ws, w.tbuf);
  p.hist = ws_ptr<uint32_t>(ws, w.hist);
  p.counters = ws_ptr<uint32_t>(ws, w.counters);
  p.selmeta = ws_ptr<uint32_t>(ws, w.selmeta);
  p.direct = ws_ptr<int32_t>(ws, w.direct);
  p.cand_t = ws_ptr<float>(ws, w.cand_t);
  p.cand_j = ws_ptr<int32_t>(ws, w.cand_j);
  p.band_t = ws_ptr<double>(ws, w.band_t);
  p.band_j = ws_ptr<int32_t>(ws, w.band_j);
  p.idx = idx;
  p.status = ws_ptr<uint32_t>(ws, w.status);
  p.block = block;
  const int bq = kv->batch * n_q;
  if (w.use_sbuf) {
    // The stored logits come from the one-token tensor-core full layer (h = 16 <= 64).
    p.part1_ml = ws_ptr<float>(ws, w.part1_ml);
    int chunk1 = 0;
    plan_decode_splits(kv, n_q, w, &p.splits1, &chunk1);
    e = launch_importance_sbuf(p, bq, s);
    if (e != cudaSuccess) return cuda_fail(e, "importance launch");
    e = launch_select_rest(p, kv->batch, s);
  } else if (kv->dtype == HS2_KV_BF16 && mq_eligible(n_q, h)) {
    // Several tokens per CTA (128 query rows): each K tile is read once per group.
    CUtensorMap tk;
    if (!make_tmap_2d(&tk, kv->k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kHeadDim,
                      (uint64_t)kv->batch * kv->max_len, kHeadDim * 2, 64, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B))
      return cuda_fail(cudaErrorInvalidValue, "tensor map of K");
    const int G = mq_tokens_per_cta(h);
    const int ctas_per_split = kv->batch * ((n_q + G - 1) / G);
    int splits = device_sm_count() / ctas_per_split;
    const int min_splits = (kv->max_len + 65535 - 1) / 65535 + 1;  // chunk below 65536
    if (splits < min_splits) splits = min_splits;
    int chunk = (kv->max_len + splits - 1) / splits;
    chunk = (chunk + 127) / 128 * 128;
    p.splits2 = (kv->max_len + chunk - 1) / chunk;
    p.chunk2 = chunk;
    e = launch_importance_mq(p, tk, kv->batch, s);
    if (e != cudaSuccess) return cuda_fail(e, "importance launch");
    e = launch_select_rest(p, kv->batch, s);
  } else if (kv->dtype == HS2_KV_BF16) {
    // Tensor-core importance pass: one CTA per SM per key chunk (128-key multiples).
    CUtensorMap tk;
    if (!make_tmap_2d(&tk, kv->k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kHeadDim,
                      (uint64_t)kv->batch * kv->max_len, kHeadDim * 2, 64, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B))
      return cuda_fail(cudaErrorInvalidValue, "tensor map of K");
    int splits = device_sm_count() / bq;
    if (splits < 1) splits = 1;
    int chunk = (kv->max_len + splits - 1) / splits;
    chunk = (chunk + 127) / 128 * 128;
    p.splits2 = (kv->max_len + chunk - 1) / chunk;
    p.chunk2 = chunk;
    e = launch_importance_tc(p, tk, bq, s);
    if (e != cudaSuccess) return cuda_fail(e, "importance launch");
    e = launch_select_rest(p, kv->batch, s);
  } else if (kv->dtype == HS2_KV_FP8_E4M3 && h <= 64) {
    CUtensorMap tk;
    if (!make_tmap_2d(&tk, kv->k, CU_TENSOR_MAP_DATA_TYPE_UINT8, kHeadDim,
                      (uint64_t)kv->batch * kv->max_len, kHeadDim, 128, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B))
      return cuda_fail(cudaErrorInvalidValue, "tensor map of K");
    int splits = device_sm_count() / bq;
    if (splits < 1) splits = 1;
    int chunk = (kv->max_len + splits - 1) / splits;
    chunk = (chunk + 127) / 128 * 128;
    p.splits2 = (kv->max_len + chunk - 1) / chunk;
    p.chunk2 = chunk;
    e = launch_importance_fp8(p, tk, bq, s);
    if (e != cudaSuccess) return cuda_fail(e, "importance launch");
    e = launch_select_rest(p, kv->batch, s);
  } else {
    e = launch_select(p, kv->batch, s);
  }
  return e == cudaSuccess ? HS2_OK : cuda_fail(e, "selection launch");
}

}  // namespace hs2

using namespace hs2;

// ---------------------------------------------------------------- chunked prefill
// The several-token tensor-core full layer over a chunk of up to 65536 new tokens, with
// a workspace of split partials only: [status][part_o][part_ml].  Splits are planned
// from a fixed target of CTAs (so the workspace size does not depend on the device).
constexpr int kMaxPrefillTokens = 65536;
constexpr int kPrefillCtaTarget = 296;  // about two CTAs per SM of a 148-SM part
constexpr int kMaxPrefillSplits = 32;

static hs2_status check_prefill(int batch, int n_q, int h, int max_len, int dtype) {
  if (batch < 1 || max_len < 1) return HS2_ERR_INVALID_ARGUMENT;
  if (dtype != HS2_KV_BF16) return HS2_ERR_UNSUPPORTED;
  if (h != 16 && h != 32 && h != 48 && h != 64 && h != 128) return HS2_ERR_UNSUPPORTED;
  if (n_q < 1 || n_q > kMaxPrefillTokens || n_q > max_len) return HS2_ERR_UNSUPPORTED;
  if ((long long)batch * max_len >= (1ll << 31)) return HS2_ERR_UNSUPPORTED;
  // One grid row per group of 128 / h tokens of a sequence: the grid's y extent.
  const int G = mq_tokens_per_cta(h);
  if ((long long)batch * ((n_q + G - 1) / G) > kMaxGridY) return HS2_ERR_UNSUPPORTED;
  return HS2_OK;
}

static int prefill_splits(int batch, int n_q, int h, int max_len) {
  const int G = mq_tokens_per_cta(h);
  const long long groups = (long long)batch * ((n_q + G - 1) / G);
  long long sp = (kPrefillCtaTarget + groups - 1) / groups;
  const long long by_len = ((long long)max_len + 63) / 64;
  if (sp > by_len) sp = by_len;
  if (sp > kMaxPrefillSplits) sp = kMaxPrefillSplits;
  return sp < 1 ? 1 : (int)sp;
}

struct PrefillLayout {
  int splits;
  size_t part_o, part_ml, total;
};

static PrefillLayout prefill_layout(int batch, int n_q, int h, int max_len) {
  PrefillLayout L;
  L.splits = prefill_splits(batch, n_q, h, max_len);
  const size_t rows = (size_t)batch * n_q * L.splits * h;
  L.part_o = 256;  // after the status word
  L.part_ml = align_up(L.part_o + rows * kHeadDim * sizeof(float), 256);
  L.total = align_up(L.part_ml + rows * 2 * sizeof(float), 256);
  return L;
}

extern "C" {

size_t hs2_workspace_bytes(int batch, int n_q, int h_q, int max_len, int window, int k_sel,
                           int dtype) {
  if (dtype != HS2_KV_BF16 && dtype != HS2_KV_FP8_E4M3) return 0;
  if (check_shape(batch, n_q, h_q, max_len, window, k_sel) != HS2_OK) return 0;
  WsLayout w;
  make_layout(batch, n_q, h_q, max_len, window, k_sel, dtype, &w);
  return w.total;
}

void hs2_debug_stall_waits(int mode) { g_stall_test = mode == 1 || mode == 2 ? mode : 0; }

void hs2_set_deterministic(int on) { g_deterministic = on ? 1 : 0; }

size_t hs2_workspace_lse64_offset(int batch, int n_q, int h_q, int max_len, int window,
                                  int k_sel, int dtype) {
  if (hs2_workspace_bytes(batch, n_q, h_q, max_len, window, k_sel, dtype) == 0)
    return ~(size_t)0;
  WsLayout w;
  make_layout(batch, n_q, h_q, max_len, window, k_sel, dtype, &w);
  return w.lse64;
}

hs2_status hs2_full_attn(const void* q, int n_q, int h_q, const hs2_kv* kv, int window,
                         int k_sel, float sm_scale, float* out, float* lse, void* workspace,
                         size_t ws_bytes, hs2_stream_t stream) {
  Prepared P;
  hs2_status st = prepare(q, n_q, h_q, kv, window, k_sel, workspace, ws_bytes, &P);
  if (st != HS2_OK) return st;
  if (!out || !aligned16(out)) return HS2_ERR_INVALID_ARGUMENT;
  return run_full(q, n_q, h_q, kv, window, k_sel, sm_scale, out, lse, workspace, P.w,
                  (cudaStream_t)stream);
}

hs2_status hs2_select(const void* q, int n_q, int h_q, const hs2_kv* kv, int window,
                      int k_sel, float sm_scale, int32_t* idx, void* workspace,
                      size_t ws_bytes, hs2_stream_t stream) {
  Prepared P;
  hs2_status st = prepare(q, n_q, h_q, kv, window, k_sel, workspace, ws_bytes, &P);
  if (st != HS2_OK) return st;
  if (!idx) return HS2_ERR_INVALID_ARGUMENT;
  return run_select(q, n_q, h_q, kv, window, k_sel, sm_scale, idx, workspace, P.w,
                    (cudaStream_t)stream);
}

hs2_status hs2_full_attn_select(const void* q, int n_q, int h_q, const hs2_kv* kv,
                                int window, int k_sel, float sm_scale, float* out,
                                int32_t* idx, float* lse, void* workspace, size_t ws_bytes,
                                hs2_stream_t stream) {
  Prepared P;
  hs2_status st = prepare(q, n_q, h_q, kv, window, k_sel, workspace, ws_bytes, &P);
  if (st != HS2_OK) return st;
  if (!out || !aligned16(out) || !idx) return HS2_ERR_INVALID_ARGUMENT;
  if (fused_full_layer(kv, n_q, h_q))  // one launch: full layer, merge and selection
    return run_full(q, n_q, h_q, kv, window, k_sel, sm_scale, out, lse, workspace, P.w,
                    (cudaStream_t)stream, idx);
  st = run_full(q, n_q, h_q, kv, window, k_sel, sm_scale, out, lse, workspace, P.w,
                (cudaStream_t)stream);
  if (st != HS2_OK) return st;
  return run_select(q, n_q, h_q, kv, window, k_sel, sm_scale, idx, workspace, P.w,
                    (cudaStream_t)stream);
}

// Block-level selection: whole blocks of `block` positions, k_sel a multiple of block,
// at most 1024 blocks kept, and the per-block keys of a row in the kernel's shared memory.
static hs2_status check_blocks(const hs2_kv* kv, int h, int k_sel, int block) {
  if (block < 2 || k_sel % block != 0) return HS2_ERR_UNSUPPORTED;
  if (k_sel / block > 1024) return HS2_ERR_UNSUPPORTED;
  if (select_blocks_smem(h, kv->max_len, block) > 200u * 1024u) return HS2_ERR_UNSUPPORTED;
  return HS2_OK;
}

hs2_status hs2_select_blocks(const void* q, int n_q, int h_q, const hs2_kv* kv, int window,
                             int k_sel, int block, float sm_scale, int32_t* idx,
                             void* workspace, size_t ws_bytes, hs2_stream_t stream) {
  Prepared P;
  hs2_status st = prepare(q, n_q, h_q, kv, window, k_sel, workspace, ws_bytes, &P);
  if (st != HS2_OK) return st;
  st = check_blocks(kv, h_q, k_sel, block);
  if (st != HS2_OK) return st;
  if (!idx) return HS2_ERR_INVALID_ARGUMENT;
  return run_select(q, n_q, h_q, kv, window, k_sel, sm_scale, idx, workspace, P.w,
                    (cudaStream_t)stream, block);
}

hs2_status hs2_full_attn_select_blocks(const void* q, int n_q, int h_q, const hs2_kv* kv,
                                       int window, int k_sel, int block, float sm_scale,
                                       float* out, int32_t* idx, float* lse, void* workspace,
                                       size_t ws_bytes, hs2_stream_t stream) {
  Prepared P;
  hs2_status st = prepare(q, n_q, h_q, kv, window, k_sel, workspace, ws_bytes, &P);
  if (st != HS2_OK) return st;
  st = check_blocks(kv, h_q, k_sel, block);
  if (st != HS2_OK) return st;
  if (!out || !aligned16(out) || !idx) return HS2_ERR_INVALID_ARGUMENT;
  st = run_full(q, n_q, h_q, kv, window, k_sel, sm_scale, out, lse, workspace, P.w,
                (cudaStream_t)stream);
  if (st != HS2_OK) return st;
  return run_select(q, n_q, h_q, kv, window, k_sel, sm_scale, idx, workspace, P.w,
                    (cudaStream_t)stream, block);
}

hs2_status hs2_sparse_attn(const void* q_layer, int n_q, int h_q, const hs2_kv* kv,
                           const int32_t* idx, int idx_width, float sm_scale, float* out,
                           void* workspace, size_t ws_bytes, hs2_stream_t stream) {
  hs2_status st = check_kv(kv);
  if (st != HS2_OK) return st;
  if (idx_width < 1 || idx_width > kMaxIdxWidth) return HS2_ERR_UNSUPPORTED;
  st = check_shape(kv->batch, n_q, h_q, kv->max_len, 1, 1);
  if (st != HS2_OK) return st;
  if (!q_layer || !idx || !out || !workspace) return HS2_ERR_INVALID_ARGUMENT;
  if (!aligned16(q_layer) || !aligned16(out) || !aligned16(workspace))
    return HS2_ERR_INVALID_ARGUMENT;
  WsLayout w;
  make_layout(kv->batch, n_q, h_q, kv->max_len, 1, 1, kv->dtype, &w);
  if (ws_bytes < sparse_prefix_bytes(w)) return HS2_ERR_WORKSPACE_TOO_SMALL;
  if (h_q <= 64) {
    // Tensor-core gather attention: the row's 128-entry tiles spread over one
    // thread-block cluster, whose CTAs merge their partials on chip and write `out`.
    FullParams f;
    f.q = static_cast<const uint16_t*>(q_layer);
    f.kv = view_of(kv);
    f.n_q = n_q;
    f.h = h_q;
    f.window = 0;
    f.k_sel = 0;
    f.sm_scale = sm_scale;
    f.chunk1 = 0;   // planned by the launcher
    f.splits1 = 0;
    f.part_o = nullptr;
    f.part_ml = nullptr;
    f.status = ws_ptr<uint32_t>(workspace, w.status);
    f.idx = idx;
    f.idx_width = idx_width;
    f.out = out;
    cudaError_t e = kv->dtype == HS2_KV_FP8_E4M3
                        ? launch_sparse_attn_fp8(f, kv->batch * n_q, (cudaStream_t)stream)
                        : launch_sparse_attn_tc(f, kv->batch * n_q, (cudaStream_t)stream);
    return e == cudaSuccess ? HS2_OK : cuda_fail(e, "sparse-attention launch");
  }
  SparseParams p;
  p.q = static_cast<const uint16_t*>(q_layer);
  p.kv = view_of(kv);
  p.idx = idx;
  p.n_q = n_q;
  p.h = h_q;
  p.idx_width = idx_width;
  p.sm_scale = sm_scale;
  p.splits4 = plan_splits4(idx_width);
  p.chunk4 = kChunk4;
  p.part_o = ws_ptr<float>(workspace, w.part4_o);
  p.part_ml = ws_ptr<float>(workspace, w.part4_ml);
  p.status = ws_ptr<uint32_t>(workspace, w.status);
  cudaError_t e = launch_sparse_attn(p, kv->batch, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "sparse-attention launch");
  MergeParams m;
  m.part_o = p.part_o;
  m.part_ml = p.part_ml;
  m.splits = p.splits4;
  m.h = h_q;
  m.out = out;
  m.lse_out = nullptr;
  m.lse64 = nullptr;
  e = launch_merge(m, kv->batch * n_q, false, (cudaStream_t)stream);
  return e == cudaSuccess ? HS2_OK : cuda_fail(e, "sparse-attention merge launch");
}

hs2_status hs2_check_device_status(void* workspace, hs2_stream_t stream) {
  if (!workspace) return HS2_ERR_INVALID_ARGUMENT;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  uint32_t word = 0;
  e = cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  if (word == 0) return HS2_OK;
  e = cudaMemsetAsync(workspace, 0, sizeof(word), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "status clear");
  for (int c = 1; c < 32; ++c)
    if (word & (1u << c)) return (hs2_status)c;
  return HS2_OK;
}

const char* hs2_status_string(hs2_status s) {
  switch (s) {
    case HS2_OK: return "ok";
    case HS2_ERR_INVALID_ARGUMENT: return "invalid argument";
    case HS2_ERR_UNSUPPORTED: return "unsupported size or type";
    case HS2_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case HS2_ERR_CUDA: return "CUDA runtime error";
    case HS2_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case HS2_ERR_INDEX_OUT_OF_RANGE: return "sparse index out of range";
    case HS2_ERR_BAD_LENGTH: return "sequence length out of range";
  }
  return "unknown status";
}

const char* hs2_last_cuda_error(void) { return g_last_cuda_error; }

int hs2_select_fused(int n_q, int h_q, int dtype) {
  hs2_kv kv;
  memset(&kv, 0, sizeof(kv));
  kv.dtype = dtype;
  if (dtype != HS2_KV_BF16 && dtype != HS2_KV_FP8_E4M3) return 0;
  if (n_q < 1 || n_q > kMaxNq || h_q < 16 || h_q > kMaxHeads || h_q % 16 != 0) return 0;
  return fused_full_layer(&kv, n_q, h_q) ? 1 : 0;
}

int hs2_abi_version(void) { return HS2_ABI_VERSION; }

hs2_status hs2_kv_append(const void* k_new, const void* v_new, int n_new, const hs2_kv* kv,
                         int32_t* lens, void* workspace, size_t ws_bytes, hs2_stream_t stream) {
  hs2_status st = check_kv(kv);
  if (st != HS2_OK) return st;
  if (!k_new || !v_new || !lens || !workspace) return HS2_ERR_INVALID_ARGUMENT;
  if (n_new < 1 || n_new > kMaxNq) return HS2_ERR_UNSUPPORTED;
  if (kv->batch < 1 || kv->max_len < 1) return HS2_ERR_INVALID_ARGUMENT;
  if ((long long)kv->batch * kv->max_len >= (1ll << 31)) return HS2_ERR_UNSUPPORTED;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(workspace))
    return HS2_ERR_INVALID_ARGUMENT;
  if (ws_bytes < 256) return HS2_ERR_WORKSPACE_TOO_SMALL;  // the status word
  AppendParams p;
  p.k_new = static_cast<const uint16_t*>(k_new);
  p.v_new = static_cast<const uint16_t*>(v_new);
  p.k = const_cast<void*>(kv->k);
  p.v = const_cast<void*>(kv->v);
  p.k_scale = const_cast<float*>(kv->k_scale);
  p.v_scale = const_cast<float*>(kv->v_scale);
  p.lens = lens;
  p.max_len = kv->max_len;
  p.n_new = n_new;
  p.fp8 = kv->dtype == HS2_KV_FP8_E4M3;
  p.status = static_cast<uint32_t*>(workspace);
  cudaError_t e = launch_kv_append(p, kv->batch, (cudaStream_t)stream);
  return e == cudaSuccess ? HS2_OK : cuda_fail(e, "kv-append launch");
}

size_t hs2_prefill_workspace_bytes(int batch, int n_q, int h_q, int max_len, int dtype) {
  if (check_prefill(batch, n_q, h_q, max_len, dtype) != HS2_OK) return 0;
  return prefill_layout(batch, n_q, h_q, max_len).total;
}

hs2_status hs2_prefill_attn(const void* q, int n_q, int h_q, const hs2_kv* kv, float sm_scale,
                            float* out, float* lse, void* workspace, size_t ws_bytes,
                            hs2_stream_t stream) {
  hs2_status st = check_kv(kv);
  if (st != HS2_OK) return st;
  st = check_prefill(kv->batch, n_q, h_q, kv->max_len, kv->dtype);
  if (st != HS2_OK) return st;
  if (!q || !out || !workspace) return HS2_ERR_INVALID_ARGUMENT;
  if (!aligned16(q) || !aligned16(out) || !aligned16(workspace)) return HS2_ERR_INVALID_ARGUMENT;
  const PrefillLayout W = prefill_layout(kv->batch, n_q, h_q, kv->max_len);
  if (ws_bytes < W.total) return HS2_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = (cudaStream_t)stream;
  FullParams p;
  p.q = static_cast<const uint16_t*>(q);
  p.kv = view_of(kv);
  p.n_q = n_q;
  p.h = h_q;
  p.window = 1;
  p.k_sel = 1;
  p.sm_scale = sm_scale;
  int chunk = (kv->max_len + W.splits - 1) / W.splits;
  chunk = (chunk + 63) / 64 * 64;
  p.splits1 = (kv->max_len + chunk - 1) / chunk;
  p.chunk1 = chunk;
  p.part_o = ws_ptr<float>(workspace, W.part_o);
  p.part_ml = ws_ptr<float>(workspace, W.part_ml);
  p.status = ws_ptr<uint32_t>(workspace, 0);
  CUtensorMap tk, tv;
  const uint64_t rows = (uint64_t)kv->batch * kv->max_len;
  if (!make_tmap_2d(&tk, kv->k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kHeadDim, rows, kHeadDim * 2,
                    64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_2d(&tv, kv->v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kHeadDim, rows, kHeadDim * 2,
                    64, 64, CU_TENSOR_MAP_SWIZZLE_128B))
    return cuda_fail(cudaErrorInvalidValue, "tensor maps of K/V");
  cudaError_t e = launch_full_attn_mq(p, tk, tv, kv->batch, s);
  if (e != cudaSuccess) return cuda_fail(e, "prefill launch");
  MergeParams m;
  m.part_o = p.part_o;
  m.part_ml = p.part_ml;
  m.splits = p.splits1;
  m.h = h_q;
  m.out = out;
  m.lse_out = lse;
  m.lse64 = nullptr;
  e = launch_merge(m, kv->batch * n_q, true, s);
  return e == cudaSuccess ? HS2_OK : cuda_fail(e, "prefill merge launch");
}

}  // extern "C"
