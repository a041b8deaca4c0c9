// Internal declarations shared by the libhs2 translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>
#include <stddef.h>

#include "../../include/hs2.h"

namespace hs2 {

constexpr int kHeadDim = 128;
constexpr int kHistBins = 4096;         // first-level radix histogram: top 12 bits
constexpr int kHistShift = 20;
constexpr int kChunk3Keys = 8192;      // keys per CTA of the compaction pass
constexpr int kMaxIdxWidth = 4096;      // window + k_sel
constexpr int kMaxNq = 64;
constexpr int kMaxHeads = 128;
constexpr long long kStallTestCycles = 20000;  // the stall test's wait limit
constexpr int kTileRing = 8;      // slots of a full-layer CTA's tile-index ring
constexpr int kRowTileSlot = 7;   // rowsync word: the row's next free tile (fused full layer)
constexpr int kSmCountBound = 160;      // workspace sizing assumes at most this many SMs

// Status bits kept in the workspace's status word (one bit per hs2_status code).
__host__ __device__ constexpr uint32_t status_bit(hs2_status s) { return 1u << (int)s; }

// ---------------------------------------------------------------------------
// Workspace layout.  Every region starts on a 256-byte boundary.
// ---------------------------------------------------------------------------
struct WsLayout {
  int bq = 0, h = 0, max_len = 0, window = 0, k_sel = 0;
  int splits1 = 0;   // key chunks per (sequence, query token) in the full layer
  int splits4 = 0;   // index chunks per (sequence, query token) in a sparse layer
  size_t status = 0;      // u32 status word; never cleared by a compute call
  size_t clear_begin = 0; // [clear_begin, clear_end) is zeroed by every full-layer call
  size_t hist = 0;        // u32 [bq][kHistBins]
  size_t rowmax = 0;      // u32 [bq][kMaxHeads] per-head maxima of a row's split partials (fused tail)
  size_t counters = 0;    // u32 [bq][8]: 0 direct, 1 cand, 2 band
  size_t clear_end = 0;
  size_t selmeta = 0;     // u32 [bq][4]: bin, eps bits, k_eff, n_c
  size_t part1_o = 0;     // f32 [bq][splits1][h][128]
  size_t part1_ml = 0;    // f32 [bq][splits1][h][2]
  size_t lse64 = 0;       // f64 [bq][h]
  size_t tbuf = 0;        // f32 [bq][max_len]  selection keys t_j
  size_t sbuf = 0;        // f32 [bq][max_len][h] raw logits (0 bytes when not used)
  bool use_sbuf = false;
  size_t direct = 0;      // i32 [bq][k_sel]
  size_t cand_t = 0;      // f32 [bq][max_len rounded up to 32]
  size_t cand_j = 0;      // i32 [bq][max_len rounded up to 32]
  size_t band_t = 0;      // f64 [bq][max_len]
  size_t band_j = 0;      // i32 [bq][max_len]
  size_t ubuf = 0;        // f32 [bq][ld_u] per-key selection bounds of the fused tail
  size_t rowcnt = 0;      // u32 [bq][kSmCountBound] per-CTA counts of the fused tail
  int ld_u = 0;           // max_len rounded up to 32
  size_t part4_o = 0;     // f32 [bq][splits4][h][128]
  size_t part4_ml = 0;    // f32 [bq][splits4][h][2]
  size_t total = 0;
};

int plan_splits1(int bq, int max_len, int num_sms);
int device_sm_count();
int plan_splits4(int idx_width);
bool make_layout(int batch, int n_q, int h, int max_len, int window, int k_sel, int dtype,
                 WsLayout* L);

template <typename T>
inline T* ws_ptr(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

// ---------------------------------------------------------------------------
// Kernel parameter blocks.
// ---------------------------------------------------------------------------
struct KvView {
  const void* k;
  const void* v;
  const float* k_scale;
  const float* v_scale;
  const int32_t* lens;
  int batch, max_len;
  int fp8;
};

struct FullParams {
  const uint16_t* q;  // bf16 bits [B][n_q][h][128]
  KvView kv;
  int n_q, h, window, k_sel;
  float sm_scale;
  int splits1, chunk1;
  float* part_o;   // [bq][splits1][h][128] unnormalised
  float* part_ml;  // [bq][splits1][h][2]: reference m, sum l
  uint32_t* status;
  const int32_t* idx = nullptr;  // gather mode (a sparse layer): [bq][idx_width] positions
  int idx_width = 0;
  float* sbuf = nullptr;          // if set: raw float32 logits of the keys outside the window
  // Gather mode only: if set, the splits1 CTAs of one row form a thread-block cluster,
  // merge their partials through distributed shared memory and write the normalised
  // output [bq][h][128] here (part_o / part_ml are then unused).
  // Full layer with a fused tail (fuse >= 1): the merged output [bq][h][128].
  float* out = nullptr;
  // Fused tail of the one-token tensor-core full layer (not gather mode):
  //   fuse 1: the CTAs of a row merge their split partials themselves into out, lse_out
  //           and lse64 (no separate merge kernel);
  //   fuse 2: the same, plus the token selection of the row into sel_idx.
  int fuse = 0;
  // Test hook for the bounded waits (hs2_debug_stall_waits): 1 = the bf16 one-token kernel
  // issues no loads or MMAs and its softmax warps' first wait gives up after
  // kStallTestCycles; 2 = the fused tail's row barriers wait for one CTA more than the row
  // has, each giving up after kStallTestCycles.
  int stall_test = 0;
  // Static key chunks per CTA (hs2_set_deterministic): results bitwise-reproducible across
  // runs, at the cost of the run-time balancing of the row's tiles.
  int deterministic = 0;
  float* lse_out = nullptr;      // [bq][h] or null
  double* lse64 = nullptr;       // [bq][h]
  float* ubuf = nullptr;         // [bq][ld_u]: per-key bound u_j = max_h x_hj (log2 units)
  int ld_u = 0;
  uint32_t* uhist = nullptr;     // [bq][kHistBins]: the u histogram, then the fine one
  uint32_t* rowmax = nullptr;    // [bq][kMaxHeads]: ordered keys of the row's largest m per head
  uint32_t* rowsync = nullptr;   // [bq][8]: arrival counters, the band list's length, the next tile
  float* cand_t = nullptr;       // [bq][ld_u] candidates of long chunks, at the chunk's offset: keys ...
  int32_t* cand_j = nullptr;     // [bq][ld_u] ... and positions
  double* band_t = nullptr;      // [bq][max_len] the row's band list: float64 keys ...
  int32_t* band_j = nullptr;     // [bq][max_len] ... and positions
  uint32_t* rowcnt = nullptr;    // [bq][kSmCountBound] keys per CTA of a row in before the band ranking
  int32_t* sel_idx = nullptr;    // [bq][window + k_sel]
};

// Split merge (full layer: log2-domain partials; sparse layers: natural-log ones).
struct MergeParams {
  const float* part_o;
  const float* part_ml;
  int splits, h;
  float* out;
  float* lse_out;  // may be null
  double* lse64;   // may be null
};

struct SelectParams {
  const uint16_t* q;
  KvView kv;
  int n_q, h, window, k_sel;
  float sm_scale;
  int splits2, chunk2;   // importance pass
  int splits3, chunk3;   // compaction pass
  const double* lse64;  // per-head lse of the full layer, [bq][h]
  const float* sbuf;     // raw float32 logits written by the full layer, or null
  // With sbuf: the full layer's split partials (m in log2 units, l), from which the
  // importance pass takes the per-head lse itself instead of waiting for the merge.
  const float* part1_ml = nullptr;
  int splits1 = 0;
  float* tbuf;
  uint32_t* hist;
  uint32_t* counters;
  uint32_t* selmeta;
  int32_t* direct;
  float* cand_t;
  int32_t* cand_j;
  double* band_t;
  int32_t* band_j;
  int32_t* idx;
  uint32_t* status;
  int block = 1;  // 1: token-level selection; > 1: whole blocks of this many positions
};

// Appending new tokens (KV append with FP8 quantisation of the new rows).
struct AppendParams {
  const uint16_t* k_new;  // bf16 [B][n_new][128]
  const uint16_t* v_new;
  void* k;                 // the cache, [B][max_len][128] (bf16 or E4M3 codes)
  void* v;
  float* k_scale;          // [B][max_len] (FP8 only)
  float* v_scale;
  int32_t* lens;           // [B], read and grown by n_new
  int max_len, n_new;
  bool fp8;
  uint32_t* status;
};

struct SparseParams {
  const uint16_t* q;
  KvView kv;
  const int32_t* idx;
  int n_q, h, idx_width;
  float sm_scale;
  int splits4, chunk4;
  float* part_o;
  float* part_ml;
  uint32_t* status;
};

// Programmatic dependent launch: the kernel may be scheduled while the previous kernel
// on the stream is finishing, so every kernel does only shared-memory / TMEM set-up
// before griddep_wait() and touches global memory after it.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// The same, optionally as a cooperative launch (every CTA resident at once), for the
// kernels whose CTAs of one row wait for one another.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_coop(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                   bool cooperative, cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeCooperative;
  attr[1].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cooperative ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// The same, with the grid's x dimension grouped into thread-block clusters of
// `cluster_x` CTAs (grid.x must be a multiple of it).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block,
                                      size_t smem, int cluster_x, cudaStream_t st,
                                      Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)cluster_x;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// Launchers (each returns the launch's cudaError_t).
cudaError_t launch_full_attn(const FullParams& p, int batch, cudaStream_t s);
cudaError_t launch_select(const SelectParams& p, int batch, cudaStream_t s);
// The selection after the importance pass (compaction + finish).
cudaError_t launch_select_rest(const SelectParams& p, int batch, cudaStream_t s);
size_t select_blocks_smem(int h, int max_len, int block);
// Importance from the full layer's stored float32 logits.
cudaError_t launch_importance_sbuf(const SelectParams& p, int bq, cudaStream_t s);
// The stored-logit path applies to single-token decode with 16 heads: 64 bytes of
// logits per key instead of re-reading its K row (256 bytes bf16, 132 bytes FP8).
inline bool sbuf_eligible(int n_q, int h, int /*dtype*/) {
  return n_q == 1 && h == 16;
}
cudaError_t launch_sparse_attn(const SparseParams& p, int batch, cudaStream_t s);
cudaError_t launch_merge(const MergeParams& p, int bq, bool log2_domain, cudaStream_t s);
cudaError_t launch_kv_append(const AppendParams& p, int batch, cudaStream_t s);

// ---------------------------------------------------------------------------
// Device helpers.
// ---------------------------------------------------------------------------
#ifdef __CUDACC__

// Wait until the previous kernel on the stream has completed and its writes are visible
// (a no-op for a kernel launched without programmatic serialisation).
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Let the next kernel on the stream be scheduled (it still waits for this grid's end).
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) {
  return __uint_as_float(b << 16);
}

// OCP FP8 E4M3 ("fn") code -> float32, from the format: sign, 4-bit exponent with
// bias 7, 3-bit mantissa, exponent 0 subnormal, S.1111.111 NaN.
__device__ __forceinline__ float e4m3_to_f32(uint32_t c) {
  const uint32_t e = (c >> 3) & 0xFu, m = c & 0x7u;
  float mag;
  if (e == 0) {
    mag = (float)m * 0.001953125f;  // m * 2^-9
  } else {
    mag = __uint_as_float(((e + 120u) << 23) | (m << 20));
  }
  if ((c & 0x7Fu) == 0x7Fu) mag = __int_as_float(0x7fc00000);
  return (c & 0x80u) ? -mag : mag;
}

__device__ __forceinline__ double e4m3_to_f64(uint32_t c) {
  return (double)e4m3_to_f32(c);  // every E4M3 value is exact in float32
}

// Monotone map float -> uint32 (larger float -> larger key); NaN excluded.
__device__ __forceinline__ uint32_t ordered_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_to_float(uint32_t k) {
  const uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  return __uint_as_float(u);
}
__device__ __forceinline__ unsigned long long ordered_key64(double f) {
  const unsigned long long u = (unsigned long long)__double_as_longlong(f);
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ void set_status(uint32_t* status, hs2_status s) {
  atomicOr(status, status_bit(s));
}

// Valid length of sequence b, clamped to [n_q, max_len] (an out-of-range length
// is recorded and clamped so that no access leaves the cache).
__device__ __forceinline__ int seq_len(const KvView& kv, int b, int n_q, uint32_t* status,
                                       bool report) {
  int L = kv.lens[b];
  if (L < n_q || L > kv.max_len) {
    if (report) set_status(status, HS2_ERR_BAD_LENGTH);
    L = L < n_q ? n_q : kv.max_len;
  }
  return L;
}

// Adds a CTA's shared-memory histogram of selection keys (kHistBins bins) to its query's
// global one, skipping every bin below the bin of the CTA's own k-th largest key: the
// k-th largest key over all of the query's CTAs is at least each CTA's, and the boundary
// search only reads bins from the top down to the bin of that key.  (If the CTA holds
// fewer than k keys every non-empty bin is added.)  Threads [tid0, tid0 + NT) call it
// together; `sync` is a barrier over exactly those threads; `red` is NT + 1 words of
// shared scratch.
template <int NT, typename Sync>
__device__ __forceinline__ void flush_hist_top(const uint32_t* hist_s, uint32_t* gh, int k,
                                               int tid, uint32_t* red, Sync sync) {
  constexpr int kPer = kHistBins / NT;  // bins per thread, thread i from the top
  static_assert(kPer * NT == kHistBins && NT % 32 == 0, "whole warps, whole bins");
  const int hi_bin = kHistBins - 1 - tid * kPer;  // this thread's bins: hi_bin down
  uint32_t loc = 0;
#pragma unroll 8
  for (int u = 0; u < kPer; ++u) loc += hist_s[hi_bin - u];
  // Exclusive prefix from the top over the threads: warp scan, then the warp totals.
  const int lane = tid & 31, w = tid >> 5;
  uint32_t incl = loc;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  if (lane == 31) red[w] = incl;
  if (tid == 0) red[NT] = 0u;  // lowest bin to add (0: all)
  sync();
  uint32_t above = incl - loc;
  for (int ww = 0; ww < w; ++ww) above += red[ww];
  if (above < (uint32_t)k && (uint32_t)k <= above + loc) {
    uint32_t cum = above;
    for (int u = 0; u < kPer; ++u) {
      cum += hist_s[hi_bin - u];
      if (cum >= (uint32_t)k) {
        red[NT] = (uint32_t)(hi_bin - u);
        break;
      }
    }
  }
  sync();
  const int lowest = (int)red[NT];
  for (int e = lowest + tid; e < kHistBins; e += NT)
    if (hist_s[e]) atomicAdd(gh + e, hist_s[e]);
}

#endif  // __CUDACC__

}  // namespace hs2
