// Token-level selection of the hybrid block (web coverage of HySparse2: toolnavs
// article 2080, fr/ko paragraph on selection granularity -- the most recent
// `window` tokens are always kept, plus the top `k_sel` tokens outside the window,
// chosen from the full layer's attention scores with no trained selector).
//
// Importance of key j is max_h exp(s_hj - lse_h).  Ranking uses the monotone
// stand-in t_j = max_h (s_hj - delta_h) with delta_h = lse_h - min_h' lse_h' (a
// common shift keeps t near the logits, where float32 is finest).
//
//   1. importance pass (grid splits2 x bq): recompute the logits of every key of
//      [0, p-window] in float32, write t_j, and count the top 12 bits of t_j's
//      order-preserving key in a shared-memory histogram flushed to global memory;
//   2. compaction pass (grid splits3 x bq): find the histogram bin holding the
//      k-th largest t; keys clearly above it are kept outright, keys within the bin
//      (plus a margin eps) become candidates;
//   3. finish (one CTA per bq): exact radix select of the k-th largest float32 key
//      tau among the candidates; keys with |t - tau| <= eps are re-scored in float64
//      from the stored inputs and ranked by (t desc, position asc); the result is
//      merged with the window, sorted ascending and padded with -1.
// The float32 pass is exact whenever its keys lie within eps/2 of the true ones,
// eps = 1e-3 * max(1, |bin edges| + max_h delta_h).
#include "tile_simt.cuh"
#include "sm100.cuh"
#include "select_common.cuh"

namespace hs2 {

__device__ __forceinline__ uint64_t sm100_evict_first_policy() { return sm100::policy_evict_first(); }
__device__ __forceinline__ uint4 sm100_ld_cg_v4_hint(const void* p, uint64_t pol) {
  return sm100::ld_global_cg_v4_hint(p, pol);
}


constexpr float kEpsRel = 1e-3f;

// ----------------------------------------------------------------------------
// 1. importance + histogram
// ----------------------------------------------------------------------------
template <int H, bool FP8>
__global__ void __launch_bounds__(kThreads) importance_simt_kernel(SelectParams p) {
  extern __shared__ __align__(16) float smem[];
  SimtSmem s = carve_simt(smem, H);
  griddep_wait();
  __shared__ uint32_t hist_s[kHistBins];
  __shared__ float delta_s[kMaxHeads];
  griddep_wait();
  const int split = blockIdx.x, bq = blockIdx.y;
  const int b = bq / p.n_q, i = bq % p.n_q;
  const int L = seq_len(p.kv, b, p.n_q, p.status, false);
  const int pos = L - p.n_q + i;
  const int n_c = pos - p.window + 1;  // |[0, p - window]|
  if (n_c <= p.k_sel) return;          // every outside key is kept
  const int k0 = split * p.chunk2;
  const int k1 = min(k0 + p.chunk2, n_c);
  if (k0 >= k1) return;

  for (int e = threadIdx.x; e < kHistBins; e += kThreads) hist_s[e] = 0u;
  load_delta(p.lse64 + (size_t)bq * H, H, delta_s, nullptr);
  load_q_scaled<H>(s.qs, p.q + (size_t)bq * H * kHeadDim, p.sm_scale);
  const size_t row_base = (size_t)b * p.kv.max_len;
  float* trow = p.tbuf + (size_t)bq * p.kv.max_len;
  for (int j0 = k0; j0 < k1; j0 += kTile) {
    __syncthreads();
    if (threadIdx.x < kTile) {
      const int j = j0 + threadIdx.x;
      s.rowidx[threadIdx.x] = j < k1 ? (int)(row_base + j) : -1;
    }
    __syncthreads();
    load_rows<FP8>(s.ks, kKsLd, p.kv.k, p.kv.k_scale, s.rowidx);
    __syncthreads();
    qk_tile<H>(s);
    __syncthreads();
    if (threadIdx.x < kTile && s.rowidx[threadIdx.x] >= 0) {
      float t = -INFINITY;
#pragma unroll 8
      for (int hd = 0; hd < H; ++hd) t = fmaxf(t, s.S[hd * kTile + threadIdx.x] - delta_s[hd]);
      trow[j0 + threadIdx.x] = t;
      atomicAdd(&hist_s[ordered_key(t) >> kHistShift], 1u);
    }
  }
  __syncthreads();
  __shared__ uint32_t flush_red[kThreads + 1];
  flush_hist_top<kThreads>(hist_s, p.hist + (size_t)bq * kHistBins, p.k_sel, threadIdx.x,
                           flush_red, [] { __syncthreads(); });
}

// Per-head shift delta_h = lse_h - min lse from the full layer's split partials (m in
// log2 units, l): M = max m over non-empty splits, lse = (M + log2 sum_s l_s 2^(m_s - M))
// ln 2, in float32 (the selection keys are float32 anyway and tolerate ~1e-6 here; the
// exact re-scoring takes the float64 lse of the merge).  One load pass, through L2.
template <int H>
__device__ __forceinline__ void delta_from_partials(const float* pml, int S, float* delta_s) {
  constexpr int kMaxS = 64;  // up to 64 splits per query (two per lane)
  __shared__ float lse_s[H];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int h = w; h < H; h += nw) {
    float2 v[kMaxS / 32];
#pragma unroll
    for (int u = 0; u < kMaxS / 32; ++u) {
      const int sp = lane + 32 * u;
      v[u] = sp < S ? __ldcg(reinterpret_cast<const float2*>(pml + ((size_t)sp * H + h) * 2))
                    : make_float2(-INFINITY, 0.f);
    }
    float M = -INFINITY;
#pragma unroll
    for (int u = 0; u < kMaxS / 32; ++u)
      if (v[u].y > 0.f) M = fmaxf(M, v[u].x);
    for (int sp = lane + kMaxS; sp < S; sp += 32) {  // rare: more than 64 splits
      const float2 x = __ldcg(reinterpret_cast<const float2*>(pml + ((size_t)sp * H + h) * 2));
      if (x.y > 0.f) M = fmaxf(M, x.x);
    }
    M = warp_max(M);
    float Ls = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int u = 0; u < kMaxS / 32; ++u)
        if (v[u].y > 0.f) Ls += v[u].y * exp2f(v[u].x - M);
      for (int sp = lane + kMaxS; sp < S; sp += 32) {
        const float2 x = __ldcg(reinterpret_cast<const float2*>(pml + ((size_t)sp * H + h) * 2));
        if (x.y > 0.f) Ls += x.y * exp2f(x.x - M);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, o);
    if (lane == 0) lse_s[h] = Ls > 0.f ? (M + __log2f(Ls)) * 0.6931471805599453f : -INFINITY;
  }
  __syncthreads();
  if (threadIdx.x < H) {
    float mn = INFINITY;
#pragma unroll
    for (int h = 0; h < H; ++h) mn = fminf(mn, lse_s[h]);
    delta_s[threadIdx.x] = lse_s[threadIdx.x] - mn;
  }
  __syncthreads();
}

// 1'. importance from the full layer's stored float32 logits (single-token decode,
//     16 heads): the same t_j and histogram without reading K again.  This pass does
//     not use the merge kernel's output (it takes the per-head lse from the partials), so
//     it waits for the previous grid (the merge, which lets it start as soon as the full
//     layer is done) only before it exits: the passes after it may read the merge's lse.
//     Everything it reads was written by the full layer and is loaded through L2.
constexpr int kSbufChunk = 4096;

template <int H>
__global__ void __launch_bounds__(kThreads) importance_sbuf_kernel(SelectParams p) {
  __shared__ uint32_t hist_s[kHistBins];
  __shared__ float delta_s[kMaxHeads];
  const int split = blockIdx.x, bq = blockIdx.y;
  const int b = bq / p.n_q, i = bq % p.n_q;
  const int L = seq_len(p.kv, b, p.n_q, p.status, false);
  const int pos = L - p.n_q + i;
  const int n_c = pos - p.window + 1;
  const int k0 = split * kSbufChunk;
  const int k1 = min(k0 + kSbufChunk, n_c);
  if (n_c <= p.k_sel || k0 >= k1) {
    griddep_wait();
    return;
  }
  for (int e = threadIdx.x; e < kHistBins; e += kThreads) hist_s[e] = 0u;
  const uint64_t pol = sm100_evict_first_policy();
  const float* __restrict__ src = p.sbuf + (size_t)bq * p.kv.max_len * H;
  float* __restrict__ trow = p.tbuf + (size_t)bq * p.kv.max_len;
  const float sc = p.sm_scale;
  // Keys are loaded kBatch at a time, all before the first is used (kBatch x H
  // floats in flight per thread): one memory round trip per kBatch keys.  The first
  // batch is requested before the shifts are computed.
  constexpr int kPer = kSbufChunk / kThreads;
  static_assert(kPer * kThreads == kSbufChunk, "chunk is a multiple of the block");
  constexpr int kBatch = 4;
  uint4 v[kBatch][H / 4];
  auto load_batch = [&](int u0) {
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int j = k0 + (u0 + u) * kThreads + threadIdx.x;
#pragma unroll
      for (int c = 0; c < H / 4; ++c)
        v[u][c] = j < k1 ? sm100_ld_cg_v4_hint(src + (size_t)j * H + 4 * c, pol)
                         : make_uint4(0, 0, 0, 0);
    }
  };
  load_batch(0);
  delta_from_partials<H>(p.part1_ml + (size_t)bq * p.splits1 * H * 2, p.splits1, delta_s);
#pragma unroll 1
  for (int u0 = 0; u0 < kPer; u0 += kBatch) {
    if (u0 > 0) load_batch(u0);
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int j = k0 + (u0 + u) * kThreads + threadIdx.x;
      if (j >= k1) continue;
      float t = -INFINITY;
#pragma unroll
      for (int c = 0; c < H / 4; ++c) {
        t = fmaxf(t, __uint_as_float(v[u][c].x) * sc - delta_s[4 * c]);
        t = fmaxf(t, __uint_as_float(v[u][c].y) * sc - delta_s[4 * c + 1]);
        t = fmaxf(t, __uint_as_float(v[u][c].z) * sc - delta_s[4 * c + 2]);
        t = fmaxf(t, __uint_as_float(v[u][c].w) * sc - delta_s[4 * c + 3]);
      }
      trow[j] = t;
      const uint32_t bin = ordered_key(t) >> kHistShift;
      atomicAdd(&hist_s[bin], 1u);
    }
  }
  __syncthreads();
  __shared__ uint32_t flush_red[kThreads + 1];
  flush_hist_top<kThreads>(hist_s, p.hist + (size_t)bq * kHistBins, p.k_sel, threadIdx.x,
                           flush_red, [] { __syncthreads(); });
  griddep_wait();
}

cudaError_t launch_importance_sbuf(const SelectParams& p, int bq, cudaStream_t st) {
  const dim3 grid((p.kv.max_len + kSbufChunk - 1) / kSbufChunk, bq);
  switch (p.h) {
    case 16: return launch_pdl(importance_sbuf_kernel<16>, grid, dim3(kThreads), 0, st, p);
    default: return cudaErrorInvalidValue;
  }
}

// ----------------------------------------------------------------------------
// 2. compaction
// ----------------------------------------------------------------------------
struct BoundaryBin {
  uint32_t bin;
  float lo, hi, eps;
};

// Every CTA of a bq finds the same boundary bin from the global histogram: thread t
// sums 16 bins, warp 0 turns the 256 sums into counts "above" (a prefix sum from the
// top bin down), and the thread whose range holds the k-th largest scans its bins.
constexpr int kBinsPerThread = kHistBins / kThreads;  // 16

__device__ __forceinline__ void load_hist_slice(const uint32_t* gh, uint32_t (&c)[kBinsPerThread]) {
  const uint4* src = reinterpret_cast<const uint4*>(gh + threadIdx.x * kBinsPerThread);
#pragma unroll
  for (int e = 0; e < kBinsPerThread / 4; ++e) {
    const uint4 v = __ldcg(src + e);
    c[4 * e] = v.x;
    c[4 * e + 1] = v.y;
    c[4 * e + 2] = v.z;
    c[4 * e + 3] = v.w;
  }
}

// c: this thread's 16 bins of the histogram (load_hist_slice), requested early.
__device__ BoundaryBin find_boundary_bin(const uint32_t (&c)[kBinsPerThread], int k_eff,
                                         float delta_max) {
  __shared__ uint32_t part[kThreads];  // indexed from the top: part[255 - t]
  __shared__ uint32_t bin_s;
  constexpr int per = kBinsPerThread;
  if (threadIdx.x == 0) bin_s = 0u;
  uint32_t loc = 0;
#pragma unroll
  for (int e = 0; e < per; ++e) loc += c[e];
  part[kThreads - 1 - threadIdx.x] = loc;
  __syncthreads();
  if (threadIdx.x < 32) {
    // lane l owns part[8l .. 8l+7]; exclusive prefix from the top
    uint32_t v[8], sum = 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      v[u] = part[8 * threadIdx.x + u];
      sum += v[u];
    }
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
      if ((int)threadIdx.x >= o) incl += x;
    }
    uint32_t run = incl - sum;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const uint32_t here = v[u];
      part[8 * threadIdx.x + u] = run;  // count strictly above this thread's range
      run += here;
    }
  }
  __syncthreads();
  const uint32_t a = part[kThreads - 1 - threadIdx.x];
  if (a < (uint32_t)k_eff && (uint32_t)k_eff <= a + loc) {
    uint32_t cum = a;
#pragma unroll
    for (int e = per - 1; e >= 0; --e) {
      if (cum + c[e] >= (uint32_t)k_eff) {
        bin_s = threadIdx.x * per + e;
        break;
      }
      cum += c[e];
    }
  }
  __syncthreads();
  BoundaryBin r;
  r.bin = bin_s;
  r.lo = key_to_float(r.bin << kHistShift);
  r.hi = key_to_float((r.bin << kHistShift) | ((1u << kHistShift) - 1u));
  // Margin around the boundary bin: the float32 logits (tensor-core accumulation) and
  // the float32 shift are far inside 1e-3 of |t| + max delta for any sane input.
  const float edge = fmaxf(fabsf(r.lo), fabsf(r.hi));
  r.eps = kEpsRel * fmaxf(1.f, edge + delta_max);
  return r;
}

// Exclusive prefix sum over the block of one value per thread; *total gets the sum.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* total) {
  __shared__ uint32_t warp_tot[kThreads / 32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  if (lane == 31) warp_tot[w] = incl;
  __syncthreads();
  uint32_t before = 0, all = 0;
#pragma unroll
  for (int k = 0; k < kThreads / 32; ++k) {
    const uint32_t c = warp_tot[k];
    before += k < w ? c : 0u;
    all += c;
  }
  __syncthreads();  // warp_tot may be reused by the next call
  *total = all;
  return before + incl - v;
}

// Each CTA takes kChunk3Keys keys of one query: kPer consecutive keys per thread,
// loaded (with the histogram) before the boundary bin is known.  Keys are sorted into
// the direct list (clearly above the boundary bin) and the candidate list (inside it,
// with the margin); the CTA counts both, reserves its ranges with one atomic per list
// and writes them, so no key waits on a global atomic.
__global__ void __launch_bounds__(kThreads) select_compact_kernel(SelectParams p) {
  constexpr int kPer = kChunk3Keys / kThreads;
  griddep_wait();
  const int split = blockIdx.x, bq = blockIdx.y;
  const int b = bq / p.n_q, i = bq % p.n_q;
  const int L = seq_len(p.kv, b, p.n_q, p.status, false);
  const int pos = L - p.n_q + i;
  const int n_c = pos - p.window + 1;
  if (n_c <= p.k_sel) return;
  const int k0 = split * kChunk3Keys;
  const int k1 = min(k0 + kChunk3Keys, n_c);
  if (k0 >= k1) return;
  const int k_eff = p.k_sel;
  const float* __restrict__ trow = p.tbuf + (size_t)bq * p.kv.max_len;
  const int j0 = k0 + threadIdx.x * kPer;
  float t[kPer];
  if (j0 + kPer <= k1 && (reinterpret_cast<uintptr_t>(trow + j0) & 15u) == 0) {
#pragma unroll
    for (int u = 0; u < kPer / 4; ++u) {
      const float4 v = __ldcg(reinterpret_cast<const float4*>(trow + j0) + u);
      t[4 * u] = v.x;
      t[4 * u + 1] = v.y;
      t[4 * u + 2] = v.z;
      t[4 * u + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int u = 0; u < kPer; ++u) t[u] = j0 + u < k1 ? __ldcg(trow + j0 + u) : -INFINITY;
  }
  uint32_t hc[kBinsPerThread];
  load_hist_slice(p.hist + (size_t)bq * kHistBins, hc);
  __shared__ float dmax_s;
  if (threadIdx.x < 32) {
    double lo = INFINITY, hi = -INFINITY;
    for (int h = threadIdx.x; h < p.h; h += 32) {
      const double l = __ldcg(p.lse64 + (size_t)bq * p.h + h);
      lo = fmin(lo, l);
      hi = fmax(hi, l);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = fmin(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmax(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if (threadIdx.x == 0) dmax_s = (float)(hi - lo);
  }
  __syncthreads();
  const BoundaryBin bb = find_boundary_bin(hc, k_eff, dmax_s);
  if (split == 0 && threadIdx.x == 0) {
    uint32_t* meta = p.selmeta + (size_t)bq * 4;
    meta[0] = bb.bin;
    meta[1] = __float_as_uint(bb.eps);
    meta[2] = (uint32_t)k_eff;
    meta[3] = (uint32_t)n_c;
  }
  const float hi_e = bb.hi + bb.eps, lo_e = bb.lo - bb.eps;
  uint32_t nd = 0, nc = 0;
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    nd += t[u] > hi_e;
    nc += t[u] <= hi_e && t[u] >= lo_e;
  }
  uint32_t tot_d, tot_c;
  uint32_t od = block_excl_scan(nd, &tot_d);
  uint32_t oc = block_excl_scan(nc, &tot_c);
  __shared__ uint32_t base_d, base_c;
  uint32_t* cnt = p.counters + (size_t)bq * 8;
  if (threadIdx.x == 0) {
    base_d = tot_d ? atomicAdd(cnt + 0, tot_d) : 0u;
    base_c = tot_c ? atomicAdd(cnt + 1, tot_c) : 0u;
  }
  __syncthreads();
  od += base_d;
  oc += base_c;
  int32_t* direct = p.direct + (size_t)bq * p.k_sel;
  float* ct = p.cand_t + (size_t)bq * p.kv.max_len;
  int32_t* cj = p.cand_j + (size_t)bq * p.kv.max_len;
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    if (t[u] > hi_e) {
      if (od < (uint32_t)p.k_sel) direct[od] = j0 + u;
      ++od;
    } else if (t[u] >= lo_e) {
      if (oc < (uint32_t)p.kv.max_len) {
        ct[oc] = t[u];
        cj[oc] = j0 + u;
      }
      ++oc;
      // The finish re-scores the candidates near the boundary from their K rows: bring
      // the row into L2 now (a hint only).
      const size_t row = (size_t)b * p.kv.max_len + (size_t)(j0 + u);
      const char* kr = static_cast<const char*>(p.kv.k) + row * (p.kv.fp8 ? kHeadDim : 2 * kHeadDim);
      asm volatile("prefetch.global.L2 [%0];" ::"l"(kr));
      if (!p.kv.fp8) asm volatile("prefetch.global.L2 [%0];" ::"l"(kr + 128));
    }
  }
}

// ----------------------------------------------------------------------------
// 3. finish: exact select + float64 refinement + window merge + sort
// ----------------------------------------------------------------------------
constexpr int kFinThreads = 1024;
constexpr int kSmallBand = 1024;  // bands up to this size are ranked pairwise in shared memory
constexpr int kBuckets = 1024;    // counting-sort buckets of the final index set
constexpr int kCandSmem = 4096;   // candidate lists up to this size are staged in shared memory
// The final sort uses a bitmap of positions in the candidate staging area (8 bytes per
// candidate slot, 32 positions per word) when the ranked range fits in it.
constexpr int kBitmapKeys = kCandSmem * 2 * 32;
static_assert(kSmallBand * (sizeof(double) + sizeof(int)) <= kMaxIdxWidth * sizeof(int),
              "band pairs must fit the scratch area");

__host__ __device__ constexpr size_t finish_dyn_smem(int H) {
  return (size_t)H * kQLd * sizeof(uint16_t) + (size_t)kCandSmem * (sizeof(float) + sizeof(int)) +
         (size_t)(kFinThreads / 32) * kHeadDim * sizeof(double);
}


template <int H, bool FP8>
__global__ void __launch_bounds__(kFinThreads) select_finish_kernel(SelectParams p) {
  __shared__ int sel[kMaxIdxWidth];
  // One scratch area: the small band's (t, position) pairs, later the sort buffer.
  __shared__ __align__(16) unsigned char scratch[kMaxIdxWidth * sizeof(int)];
  double* band_ts = reinterpret_cast<double*>(scratch);                    // [kSmallBand]
  int* band_js = reinterpret_cast<int*>(scratch + kSmallBand * sizeof(double));
  int* tmp = reinterpret_cast<int*>(scratch);                              // [kMaxIdxWidth]
  __shared__ uint32_t bucket[kBuckets], bucket_beg[kBuckets];
  __shared__ uint32_t n_sel, n_band_s, gt_s;
  extern __shared__ __align__(16) unsigned char fin_dyn[];
  uint16_t* qsm = reinterpret_cast<uint16_t*>(fin_dyn);  // [H][kQLd] bf16 q of this query
  float* cts = reinterpret_cast<float*>(fin_dyn + (size_t)H * kQLd * sizeof(uint16_t));
  int* cjs = reinterpret_cast<int*>(cts + kCandSmem);
  float* kdsm = reinterpret_cast<float*>(cjs + kCandSmem);  // [warps][128] widened K rows
  __shared__ double dlt[H];
  griddep_wait();
  const int bq = blockIdx.x;
  const int b = bq / p.n_q, i = bq % p.n_q;
  const int L = seq_len(p.kv, b, p.n_q, p.status, false);
  const int pos = L - p.n_q + i;
  const int width = p.window + p.k_sel;
  const int n_c = pos - p.window + 1;
  int32_t* out = p.idx + (size_t)bq * width;
  if (n_c <= p.k_sel) {
    for (int e = threadIdx.x; e < width; e += blockDim.x) out[e] = e <= pos ? e : -1;
    __threadfence();  // visible before the CTA counts as done for the next kernel
    return;
  }
  // Loads that depend on nothing but the previous pass, issued together: the counts,
  // the margin, this query's q and the per-head shifts.
  const uint32_t* cnt = p.counters + (size_t)bq * 8;
  const uint32_t n_direct = min(__ldcg(cnt + 0), (uint32_t)p.k_sel);
  const uint32_t n_cand = min(__ldcg(cnt + 1), (uint32_t)p.kv.max_len);
  const float eps = __uint_as_float(__ldcg(p.selmeta + (size_t)bq * 4 + 1));
  for (int e = threadIdx.x; e < H * (kHeadDim / 8); e += blockDim.x) {
    const int h = e / (kHeadDim / 8), c = (e % (kHeadDim / 8)) * 8;
    *reinterpret_cast<uint4*>(qsm + h * kQLd + c) =
        *reinterpret_cast<const uint4*>(p.q + ((size_t)bq * H + h) * kHeadDim + c);
  }
  load_delta(p.lse64 + (size_t)bq * H, H, nullptr, dlt);  // (synchronises the block)
  const int need = p.k_sel - (int)n_direct;  // >= 1 by construction
  const float* ct = p.cand_t + (size_t)bq * p.kv.max_len;
  const int32_t* cj = p.cand_j + (size_t)bq * p.kv.max_len;
  // The direct list goes to the front of the selection; the candidates are staged in
  // shared memory when they fit.
  const bool cand_smem = n_cand <= (uint32_t)kCandSmem;
  for (uint32_t e = threadIdx.x; e < n_direct; e += blockDim.x)
    sel[e] = __ldcg(p.direct + (size_t)bq * p.k_sel + e);
  if (cand_smem)
    for (uint32_t e = threadIdx.x; e < n_cand; e += blockDim.x) {
      cts[e] = __ldcg(ct + e);
      cjs[e] = __ldcg(cj + e);
    }
  if (threadIdx.x == 0) {
    n_sel = n_direct;
    n_band_s = 0;
  }
  __syncthreads();
  auto cand_t = [&](uint32_t e) { return cand_smem ? cts[e] : __ldcg(ct + e); };
  auto cand_j = [&](uint32_t e) { return cand_smem ? cjs[e] : __ldcg(cj + e); };

  // tau: the need-th largest float32 key among the candidates (whose keys share their
  // high bits: the radix passes start below the bits that min and max have in common).
  __shared__ uint32_t kmin_s, kmax_s;
  if (threadIdx.x == 0) {
    kmin_s = 0xffffffffu;
    kmax_s = 0u;
  }
  __syncthreads();
  {
    uint32_t lo = 0xffffffffu, hi = 0u;
    for (uint32_t e = threadIdx.x; e < n_cand; e += blockDim.x) {
      const uint32_t k = ordered_key(cand_t(e));
      lo = min(lo, k);
      hi = max(hi, k);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if ((threadIdx.x & 31) == 0) {
      atomicMin(&kmin_s, lo);
      atomicMax(&kmax_s, hi);
    }
  }
  __syncthreads();
  const uint32_t tau_key = block_kth_largest<uint32_t, 32>(
      (int)n_cand, need, [&](int e) { return ordered_key(cand_t((uint32_t)e)); },
      [](int) { return true; }, &gt_s, kmin_s, kmax_s);
  const float tau = key_to_float(tau_key);
  const float hi_b = tau + eps, lo_b = tau - eps;

  // Candidates above the band are kept; band keys are listed for re-scoring (in shared
  // memory while the band is small, else in the workspace).
  int32_t* bj = p.band_j + (size_t)bq * p.kv.max_len;
  double* bt = p.band_t + (size_t)bq * p.kv.max_len;
  const uint32_t n_cand_r = (n_cand + 31u) & ~31u;  // whole warps take part in the ballots
  for (uint32_t e = threadIdx.x; e < n_cand_r; e += blockDim.x) {
    const bool in = e < n_cand;
    const float t = in ? cand_t(e) : -INFINITY;
    const int j = in ? cand_j(e) : -1;
    const bool keep = in && t > hi_b;
    const bool band = in && !keep && t >= lo_b;
    const uint32_t sk = warp_slot(keep, &n_sel);
    if (keep && sk < (uint32_t)kMaxIdxWidth) sel[sk] = j;
    const uint32_t sb = warp_slot(band, &n_band_s);
    if (band) {
      bj[sb] = j;
      if (sb < (uint32_t)kSmallBand) band_js[sb] = j;
    }
  }
  __syncthreads();
  const int n_band = (int)n_band_s;
  const int need2 = p.k_sel - (int)n_sel;  // taken from the band
  const bool band_smem = n_band <= kSmallBand;

  if (need2 > 0) {
    // float64 re-scoring of the band, one warp per key.
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float* kd = kdsm + warp * kHeadDim;
    for (int e = warp; e < n_band; e += blockDim.x / 32) {
      const int j = band_smem ? band_js[e] : __ldcg(bj + e);
      const double best =
          rescore_f64<H, FP8>(p.kv, p.sm_scale, (size_t)b * p.kv.max_len + j,
                              reinterpret_cast<const uint8_t*>(qsm), kQLd * 2, 16, dlt, kd, lane);
      if (lane == 0) {
        if (band_smem) band_ts[e] = best;
        else bt[e] = best;
      }
    }
    __syncthreads();
    if (band_smem) {
      // Small band: rank every key by (t desc, position asc) against all the others.
      for (int e = threadIdx.x; e < n_band; e += blockDim.x) {
        const double te = band_ts[e];
        const int je = band_js[e];
        int rank = 0;
        for (int f = 0; f < n_band; ++f) {
          const double tf = band_ts[f];
          rank += (tf > te) || (tf == te && band_js[f] < je);
        }
        if (rank < need2) {
          const uint32_t slot = atomicAdd(&n_sel, 1u);
          if (slot < (uint32_t)kMaxIdxWidth) sel[slot] = je;
        }
      }
    } else {
      // Boundary value among the band, then the lowest positions among its ties.
      const unsigned long long vb = block_kth_largest<unsigned long long, 64>(
          n_band, need2, [&](int e) { return ordered_key64(__ldcg(bt + e)); },
          [](int) { return true; }, &gt_s);
      const uint32_t n_gt = gt_s;
      const int take_eq = need2 - (int)n_gt;
      const uint32_t jb_inv = block_kth_largest<uint32_t, 32>(
          n_band, take_eq, [&](int e) { return ~(uint32_t)__ldcg(bj + e); },
          [&](int e) { return ordered_key64(__ldcg(bt + e)) == vb; }, &gt_s);
      const int jb = (int)~jb_inv;
      for (int e = threadIdx.x; e < n_band; e += blockDim.x) {
        const unsigned long long kk = ordered_key64(__ldcg(bt + e));
        const int je = __ldcg(bj + e);
        if (kk > vb || (kk == vb && je <= jb)) {
          const uint32_t slot = atomicAdd(&n_sel, 1u);
          if (slot < (uint32_t)kMaxIdxWidth) sel[slot] = je;
        }
      }
    }
  }
  __syncthreads();
  // Every top key lies in [0, n_c) and the forced recent window [n_c, p] lies above
  // them, already in order: only the top keys are sorted.
  const int n = (int)min(n_sel, (uint32_t)kMaxIdxWidth);
  const int n_win = pos - n_c + 1;
  if (n_c <= kBitmapKeys) {
    // Bitmap of the positions (in the candidate staging area, no longer needed): set
    // one bit per key, then each thread walks its run of words in order, starting at
    // the number of keys below the run (a block-wide prefix sum of popcounts).
    uint32_t* bm = reinterpret_cast<uint32_t*>(cts);
    const int nw = (n_c + 31) / 32;
    const int per = (nw + (int)blockDim.x - 1) / (int)blockDim.x;
    for (int e = threadIdx.x; e < nw; e += blockDim.x) bm[e] = 0u;
    __syncthreads();
    for (int e = threadIdx.x; e < n; e += blockDim.x)
      atomicOr(&bm[sel[e] >> 5], 1u << (sel[e] & 31));
    __syncthreads();
    const int w0 = threadIdx.x * per, w1 = min(w0 + per, nw);
    uint32_t cnt = 0;
    for (int w = w0; w < w1; ++w) cnt += __popc(bm[w]);
    __shared__ uint32_t warp_cnt[kFinThreads / 32];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    uint32_t incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += x;
    }
    if (lane == 31) warp_cnt[wid] = incl;
    __syncthreads();
    uint32_t base = incl - cnt;
    for (int k = 0; k < wid; ++k) base += warp_cnt[k];
    for (int w = w0; w < w1; ++w) {
      uint32_t bits = bm[w];
      while (bits) {
        const int bpos = __ffs(bits) - 1;
        bits &= bits - 1;
        if (base < (uint32_t)n) out[base] = w * 32 + bpos;
        ++base;
      }
    }
    for (int e = n + threadIdx.x; e < width; e += blockDim.x)
      out[e] = e < n + n_win ? n_c + (e - n) : -1;
  } else {
    // Counting sort on the bucket floor(position * kBuckets / n_c) (monotone; about one
    // key per bucket), then each key's rank inside its bucket.
    const float bscale = (float)kBuckets / (float)n_c;
    auto bucket_of = [&](int v) { return min(kBuckets - 1, (int)((float)v * bscale)); };
    for (int e = threadIdx.x; e < kBuckets; e += blockDim.x) bucket[e] = 0u;
    __syncthreads();
    for (int e = threadIdx.x; e < n; e += blockDim.x) atomicAdd(&bucket[bucket_of(sel[e])], 1u);
    __syncthreads();
    if (threadIdx.x < 32) {  // exclusive prefix over the buckets, 32 per lane
      const int lane = threadIdx.x;
      uint32_t sum = 0;
      for (int u = 0; u < kBuckets / 32; ++u) sum += bucket[lane * (kBuckets / 32) + u];
      uint32_t incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += x;
      }
      uint32_t run = incl - sum;
      for (int u = 0; u < kBuckets / 32; ++u) {
        const uint32_t c = bucket[lane * (kBuckets / 32) + u];
        bucket[lane * (kBuckets / 32) + u] = run;
        bucket_beg[lane * (kBuckets / 32) + u] = run;
        run += c;
      }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < n; e += blockDim.x) {
      const int v = sel[e];
      tmp[atomicAdd(&bucket[bucket_of(v)], 1u)] = v;  // bucket[b] advances to b's end
    }
    __syncthreads();
    for (int e = threadIdx.x; e < n; e += blockDim.x) {
      const int v = tmp[e];
      const int bk = bucket_of(v);
      const uint32_t beg = bucket_beg[bk], end = bucket[bk];
      uint32_t rank = 0;
      for (uint32_t x = beg; x < end; ++x) rank += tmp[x] < v;
      sel[beg + rank] = v;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < width; e += blockDim.x)
      out[e] = e < n ? sel[e] : (e < n + n_win ? n_c + (e - n) : -1);
  }
  // The index set is complete and visible: the next kernel (a sparse layer, which reads
  // it without waiting for this grid to end) may start.
  __threadfence();
  __syncthreads();
  griddep_launch_dependents();
  // Leave this query's histogram and counters at zero for the next selection.
  uint32_t* gh = p.hist + (size_t)bq * kHistBins;
  for (int e = threadIdx.x; e < kHistBins; e += blockDim.x) gh[e] = 0u;
  if (threadIdx.x < 8) p.counters[(size_t)bq * 8 + threadIdx.x] = 0u;
}

// ----------------------------------------------------------------------------
// 4. block-level selection (the first-generation scheme, a comparator)
// ----------------------------------------------------------------------------
// Positions [0, n_c) form aligned blocks of p.block positions, the last one cut at
// n_c.  A block's key is the largest float32 key t of its positions (t orders the
// positions as their importance does, and the maximum commutes with that order).
// The kb = k_sel / block best blocks are kept whole, ties to the lower block: tau is
// the kb-th largest block key; blocks above tau + eps are kept, and the blocks inside
// [tau - eps, tau + eps] get their exact score -- the float64 maximum over their
// positions of max_h(s_hj - delta_h), re-scored from the stored inputs as in the finish
// kernel -- and are ranked by (score desc, block asc).  Output: the kept blocks'
// positions in order, then the window, then -1.
constexpr int kBlkThreads = 1024;
constexpr int kBlkSmallBand = 1024;  // bands up to this size are ranked in shared memory

__host__ __device__ constexpr size_t blocks_dyn_smem(int H, int max_blocks) {
  return (size_t)H * kQLd * sizeof(uint16_t) + (size_t)(kBlkThreads / 32) * kHeadDim * sizeof(double) +
         (size_t)max_blocks * sizeof(float);
}

template <int H, bool FP8>
__global__ void __launch_bounds__(kBlkThreads) select_blocks_kernel(SelectParams p) {
  extern __shared__ __align__(16) unsigned char blk_dyn[];
  uint16_t* qsm = reinterpret_cast<uint16_t*>(blk_dyn);  // [H][kQLd] bf16 q of this query
  float* kdsm = reinterpret_cast<float*>(blk_dyn + (size_t)H * kQLd * sizeof(uint16_t));
  float* bkey = reinterpret_cast<float*>(blk_dyn + (size_t)H * kQLd * sizeof(uint16_t) +
                                         (size_t)(kBlkThreads / 32) * kHeadDim * sizeof(double));
  __shared__ double dlt[H];
  __shared__ unsigned long long band_key[kBlkSmallBand];  // exact scores, ordered keys
  __shared__ int band_blk[kBlkSmallBand];
  __shared__ int chosen[kMaxIdxWidth / 2];
  __shared__ uint32_t n_keep_s, n_band_s, gt_s;
  griddep_wait();
  const int bq = blockIdx.x;
  const int b = bq / p.n_q, i = bq % p.n_q;
  const int L = seq_len(p.kv, b, p.n_q, p.status, false);
  const int pos = L - p.n_q + i;
  const int width = p.window + p.k_sel;
  const int n_c = pos - p.window + 1;
  const int blk = p.block, kb = p.k_sel / p.block;
  const int n_blk = n_c > 0 ? (n_c + blk - 1) / blk : 0;
  int32_t* out = p.idx + (size_t)bq * width;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int kWarps = kBlkThreads / 32;
  if (n_blk > kb) {
    for (int e = threadIdx.x; e < H * (kHeadDim / 8); e += blockDim.x) {
      const int h = e / (kHeadDim / 8), c = (e % (kHeadDim / 8)) * 8;
      *reinterpret_cast<uint4*>(qsm + h * kQLd + c) =
          *reinterpret_cast<const uint4*>(p.q + ((size_t)bq * H + h) * kHeadDim + c);
    }
    load_delta(p.lse64 + (size_t)bq * H, H, nullptr, dlt);  // (synchronises the block)
    // Block keys: one thread per block, its positions read with independent 16-byte
    // loads where the row is aligned (many loads in flight instead of one per warp).
    const float* trow = p.tbuf + (size_t)bq * p.kv.max_len;
    for (int c = threadIdx.x; c < n_blk; c += blockDim.x) {
      const int j0 = c * blk, j1 = min(j0 + blk, n_c);
      float m = -INFINITY;
      int j = j0;
      if ((reinterpret_cast<uintptr_t>(trow + j0) & 15u) == 0) {
#pragma unroll 8
        for (; j + 4 <= j1; j += 4) {
          const float4 v = __ldcg(reinterpret_cast<const float4*>(trow + j));
          m = fmaxf(m, fmaxf(fmaxf(v.x, v.y), fmaxf(v.z, v.w)));
        }
      }
      for (; j < j1; ++j) m = fmaxf(m, __ldcg(trow + j));
      bkey[c] = m;
    }
    if (threadIdx.x == 0) {
      n_keep_s = 0u;
      n_band_s = 0u;
    }
    __syncthreads();
    const uint32_t tau_key = block_kth_largest<uint32_t, 32>(
        n_blk, kb, [&](int e) { return ordered_key(bkey[e]); }, [](int) { return true; }, &gt_s);
    const float tau = key_to_float(tau_key);
    double dmax = 0.0;
    for (int h = 0; h < H; ++h) dmax = fmax(dmax, dlt[h]);
    const float eps = kEpsRel * fmaxf(1.f, fabsf(tau) + (float)dmax);
    const float hi_b = tau + eps, lo_b = tau - eps;
    // Blocks above the band are kept (fewer than kb: their keys exceed the kb-th);
    // band blocks are listed for re-scoring (shared memory while the band is small,
    // else the workspace).
    int32_t* bj = p.band_j + (size_t)bq * p.kv.max_len;
    unsigned long long* bk = reinterpret_cast<unsigned long long*>(p.band_t + (size_t)bq * p.kv.max_len);
    const int n_blk_r = (n_blk + 31) & ~31;
    for (int c = threadIdx.x; c < n_blk_r; c += blockDim.x) {
      const bool in = c < n_blk;
      const float t = in ? bkey[c] : -INFINITY;
      const bool keep = in && t > hi_b;
      const bool band = in && !keep && t >= lo_b;
      const uint32_t sk = warp_slot(keep, &n_keep_s);
      if (keep && sk < (uint32_t)(kMaxIdxWidth / 2)) chosen[sk] = c;
      const uint32_t sb = warp_slot(band, &n_band_s);
      if (band) {
        bj[sb] = c;
        bk[sb] = 0ull;
        if (sb < (uint32_t)kBlkSmallBand) {
          band_blk[sb] = c;
          band_key[sb] = 0ull;
        }
      }
    }
    __syncthreads();
    const int n_band = (int)n_band_s;
    const bool band_smem = n_band <= kBlkSmallBand;
    const int need2 = kb - (int)n_keep_s;  // >= 1: tau's own block is in the band
    // float64 re-scoring of the band blocks' positions, one warp per position; each
    // block's score is the maximum over its positions (atomic max on ordered keys).
    float* kd = kdsm + warp * kHeadDim;
    const long long n_pos = (long long)n_band * blk;
    for (long long f = warp; f < n_pos; f += kWarps) {
      const int e = (int)(f / blk);
      const int c = band_smem ? band_blk[e] : __ldcg(bj + e);
      const int j = c * blk + (int)(f % blk);
      // Past the cut last block, or a position that cannot hold the block's exact
      // maximum: its float32 key is more than eps below the block's (each float32 key
      // is within eps / 2 of the exact one).  Both uniform over the warp.
      if (j >= n_c || __ldcg(trow + j) < bkey[c] - eps) continue;
      const double best =
          rescore_f64<H, FP8>(p.kv, p.sm_scale, (size_t)b * p.kv.max_len + j,
                              reinterpret_cast<const uint8_t*>(qsm), kQLd * 2, 16, dlt, kd, lane);
      if (lane == 0) {
        if (band_smem) atomicMax(&band_key[e], ordered_key64(best));
        else atomicMax(bk + e, ordered_key64(best));
      }
    }
    __syncthreads();
    if (band_smem) {
      // Small band: rank every block by (score desc, block asc) against the others.
      for (int e = threadIdx.x; e < n_band; e += blockDim.x) {
        const unsigned long long ke = band_key[e];
        const int ce = band_blk[e];
        int rank = 0;
        for (int f = 0; f < n_band; ++f) {
          const unsigned long long kf = band_key[f];
          rank += (kf > ke) || (kf == ke && band_blk[f] < ce);
        }
        if (rank < need2) chosen[atomicAdd(&n_keep_s, 1u)] = ce;
      }
    } else {
      // Boundary score among the band, then the lowest blocks among its ties.
      const unsigned long long vb = block_kth_largest<unsigned long long, 64>(
          n_band, need2, [&](int e) { return __ldcg(bk + e); }, [](int) { return true; }, &gt_s);
      const int take_eq = need2 - (int)gt_s;
      const uint32_t cb_inv = block_kth_largest<uint32_t, 32>(
          n_band, take_eq, [&](int e) { return ~(uint32_t)__ldcg(bj + e); },
          [&](int e) { return __ldcg(bk + e) == vb; }, &gt_s);
      const int cb = (int)~cb_inv;
      for (int e = threadIdx.x; e < n_band; e += blockDim.x) {
        const unsigned long long ke = __ldcg(bk + e);
        const int ce = __ldcg(bj + e);
        if (ke > vb || (ke == vb && ce <= cb)) chosen[atomicAdd(&n_keep_s, 1u)] = ce;
      }
    }
    __syncthreads();
    // kb blocks in ascending order (rank of each among the kept), then their positions:
    // every kept block is whole except possibly the cut last block, which sorts last.
    int* sorted = reinterpret_cast<int*>(band_blk);  // the band lists are no longer needed
    for (int e = threadIdx.x; e < kb; e += blockDim.x) {
      const int ce = chosen[e];
      int rank = 0;
      for (int f = 0; f < kb; ++f) rank += chosen[f] < ce;
      sorted[rank] = ce;
    }
    __syncthreads();
    const int last = sorted[kb - 1];
    const int n_sel = (kb - 1) * blk + min(blk, n_c - last * blk);
    const int n_win = pos - n_c + 1;
    for (int e = threadIdx.x; e < width; e += blockDim.x) {
      int v = -1;
      if (e < n_sel) v = sorted[e / blk] * blk + e % blk;
      else if (e < n_sel + n_win) v = n_c + (e - n_sel);
      out[e] = v;
    }
  } else {
    // No more blocks than the budget: every position of [0, pos] is kept.
    for (int e = threadIdx.x; e < width; e += blockDim.x) out[e] = e <= pos ? e : -1;
  }
  // The index set is complete and visible: the next kernel may start.
  __threadfence();
  __syncthreads();
  griddep_launch_dependents();
  // Leave this query's histogram and counters at zero for the next selection.
  uint32_t* gh = p.hist + (size_t)bq * kHistBins;
  for (int e = threadIdx.x; e < kHistBins; e += blockDim.x) gh[e] = 0u;
  if (threadIdx.x < 8) p.counters[(size_t)bq * 8 + threadIdx.x] = 0u;
}

// ----------------------------------------------------------------------------
template <int H, bool FP8>
static cudaError_t launch_rest_t(const SelectParams& p, int batch, cudaStream_t st);

template <int H, bool FP8>
static cudaError_t launch_select_t(const SelectParams& p, int batch, cudaStream_t st) {
  const size_t smem = simt_smem_bytes(H);
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(importance_simt_kernel<H, FP8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int bq = batch * p.n_q;
  cudaError_t e = launch_pdl(importance_simt_kernel<H, FP8>, dim3(p.splits2, bq), dim3(kThreads),
                             smem, st, p);
  if (e != cudaSuccess) return e;
  return launch_rest_t<H, FP8>(p, batch, st);
}

template <int H, bool FP8>
static cudaError_t launch_rest_t(const SelectParams& p, int batch, cudaStream_t st) {
  const int bq = batch * p.n_q;
  if (p.block > 1) {
    const int max_blocks = (p.kv.max_len + p.block - 1) / p.block;
    const size_t dyn = blocks_dyn_smem(H, max_blocks);
    static size_t attr_bytes = 0;
    if (dyn > attr_bytes) {
      cudaError_t e = cudaFuncSetAttribute(select_blocks_kernel<H, FP8>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
      if (e != cudaSuccess) return e;
      attr_bytes = dyn;
    }
    return launch_pdl(select_blocks_kernel<H, FP8>, dim3(bq), dim3(kBlkThreads), dyn, st, p);
  }
  cudaError_t e = launch_pdl(select_compact_kernel, dim3(p.splits3, bq), dim3(kThreads), 0, st, p);
  if (e != cudaSuccess) return e;
  const size_t dyn = finish_dyn_smem(H);
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(select_finish_kernel<H, FP8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  return launch_pdl(select_finish_kernel<H, FP8>, dim3(bq), dim3(kFinThreads), dyn, st, p);
}

template <bool FP8>
static cudaError_t launch_rest_h(const SelectParams& p, int batch, cudaStream_t st) {
  switch (p.h) {
    case 16: return launch_rest_t<16, FP8>(p, batch, st);
    case 32: return launch_rest_t<32, FP8>(p, batch, st);
    case 48: return launch_rest_t<48, FP8>(p, batch, st);
    case 64: return launch_rest_t<64, FP8>(p, batch, st);
    case 80: return launch_rest_t<80, FP8>(p, batch, st);
    case 96: return launch_rest_t<96, FP8>(p, batch, st);
    case 112: return launch_rest_t<112, FP8>(p, batch, st);
    case 128: return launch_rest_t<128, FP8>(p, batch, st);
    default: return cudaErrorInvalidValue;
  }
}

// Dynamic shared memory of the block-selection kernel for these sizes.
size_t select_blocks_smem(int h, int max_len, int block) {
  return blocks_dyn_smem(h, (max_len + block - 1) / block);
}

cudaError_t launch_select_rest(const SelectParams& p, int batch, cudaStream_t st) {
  return p.kv.fp8 ? launch_rest_h<true>(p, batch, st) : launch_rest_h<false>(p, batch, st);
}

template <bool FP8>
static cudaError_t launch_select_h(const SelectParams& p, int batch, cudaStream_t st) {
  switch (p.h) {
    case 16: return launch_select_t<16, FP8>(p, batch, st);
    case 32: return launch_select_t<32, FP8>(p, batch, st);
    case 48: return launch_select_t<48, FP8>(p, batch, st);
    case 64: return launch_select_t<64, FP8>(p, batch, st);
    case 80: return launch_select_t<80, FP8>(p, batch, st);
    case 96: return launch_select_t<96, FP8>(p, batch, st);
    case 112: return launch_select_t<112, FP8>(p, batch, st);
    case 128: return launch_select_t<128, FP8>(p, batch, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_select(const SelectParams& p, int batch, cudaStream_t st) {
  return p.kv.fp8 ? launch_select_h<true>(p, batch, st) : launch_select_h<false>(p, batch, st);
}

}  // namespace hs2
