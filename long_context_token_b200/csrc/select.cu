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
// The float32 pass is exact whenever its logits lie within eps/2 of the true ones,
// eps = 1e-3 * max(1, |bin edges|).
#include "tile_simt.cuh"

namespace hs2 {

constexpr float kEpsRel = 1e-3f;

// ----------------------------------------------------------------------------
// 1. importance + histogram
// ----------------------------------------------------------------------------
template <int H, bool FP8>
__global__ void __launch_bounds__(kThreads) importance_simt_kernel(SelectParams p) {
  extern __shared__ __align__(16) float smem[];
  SimtSmem s = carve_simt(smem, H);
  __shared__ uint32_t hist_s[kHistBins];
  __shared__ float delta_s[kMaxHeads];
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
  for (int hd = threadIdx.x; hd < H; hd += kThreads) delta_s[hd] = p.delta32[(size_t)bq * H + hd];
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
  uint32_t* gh = p.hist + (size_t)bq * kHistBins;
  for (int e = threadIdx.x; e < kHistBins; e += kThreads)
    if (hist_s[e]) atomicAdd(gh + e, hist_s[e]);
}

// ----------------------------------------------------------------------------
// 2. compaction
// ----------------------------------------------------------------------------
struct BoundaryBin {
  uint32_t bin;
  float lo, hi, eps;
};

// Every CTA of a bq finds the same boundary bin from the global histogram.
__device__ BoundaryBin find_boundary_bin(const uint32_t* gh, int k_eff) {
  __shared__ uint32_t part[kThreads];
  __shared__ uint32_t above[kThreads];
  __shared__ uint32_t bin_s;
  constexpr int per = kHistBins / kThreads;  // 16 bins per thread
  if (threadIdx.x == 0) bin_s = 0u;
  uint32_t loc = 0;
  for (int e = 0; e < per; ++e) loc += __ldcg(gh + threadIdx.x * per + e);
  part[threadIdx.x] = loc;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t cum = 0;
    for (int t = kThreads - 1; t >= 0; --t) {
      above[t] = cum;
      cum += part[t];
    }
  }
  __syncthreads();
  const uint32_t a = above[threadIdx.x];
  if (a < (uint32_t)k_eff && (uint32_t)k_eff <= a + loc) {
    uint32_t cum = a;
    for (int e = per - 1; e >= 0; --e) {
      const uint32_t bin = threadIdx.x * per + e;
      const uint32_t c = __ldcg(gh + bin);
      if (cum + c >= (uint32_t)k_eff) {
        bin_s = bin;
        break;
      }
      cum += c;
    }
  }
  __syncthreads();
  BoundaryBin r;
  r.bin = bin_s;
  r.lo = key_to_float(r.bin << kHistShift);
  r.hi = key_to_float((r.bin << kHistShift) | ((1u << kHistShift) - 1u));
  r.eps = kEpsRel * fmaxf(1.f, fmaxf(fabsf(r.lo), fabsf(r.hi)));
  return r;
}

// Warp-aggregated append of `pred` lanes to a list; returns the slot or -1.
__device__ __forceinline__ int warp_append(bool pred, uint32_t* counter) {
  const unsigned m = __ballot_sync(0xffffffffu, pred);
  if (!m) return -1;
  const int lane = threadIdx.x & 31;
  const int leader = __ffs(m) - 1;
  uint32_t base = 0;
  if (lane == leader) base = atomicAdd(counter, (uint32_t)__popc(m));
  base = __shfl_sync(0xffffffffu, base, leader);
  return pred ? (int)(base + __popc(m & ((1u << lane) - 1u))) : -1;
}

__global__ void __launch_bounds__(kThreads) select_compact_kernel(SelectParams p) {
  const int split = blockIdx.x, bq = blockIdx.y;
  const int b = bq / p.n_q, i = bq % p.n_q;
  const int L = seq_len(p.kv, b, p.n_q, p.status, false);
  const int pos = L - p.n_q + i;
  const int n_c = pos - p.window + 1;
  if (n_c <= p.k_sel) return;
  const int k_eff = p.k_sel;
  const BoundaryBin bb = find_boundary_bin(p.hist + (size_t)bq * kHistBins, k_eff);
  if (split == 0 && threadIdx.x == 0) {
    uint32_t* meta = p.selmeta + (size_t)bq * 4;
    meta[0] = bb.bin;
    meta[1] = __float_as_uint(bb.eps);
    meta[2] = (uint32_t)k_eff;
    meta[3] = (uint32_t)n_c;
  }
  const float hi_e = bb.hi + bb.eps, lo_e = bb.lo - bb.eps;
  const int k0 = split * p.chunk3;
  const int k1 = min(k0 + p.chunk3, n_c);
  const float* trow = p.tbuf + (size_t)bq * p.kv.max_len;
  uint32_t* cnt = p.counters + (size_t)bq * 8;
  int32_t* direct = p.direct + (size_t)bq * p.k_sel;
  float* ct = p.cand_t + (size_t)bq * p.kv.max_len;
  int32_t* cj = p.cand_j + (size_t)bq * p.kv.max_len;
  // Uniform trip count per warp so that every lane takes part in the ballots.
  for (int j0 = k0; j0 < k1; j0 += kThreads) {
    const int j = j0 + threadIdx.x;
    const float t = j < k1 ? __ldcg(trow + j) : -INFINITY;
    const bool is_direct = j < k1 && t > hi_e;
    const bool is_cand = j < k1 && !is_direct && t >= lo_e;
    const int sd = warp_append(is_direct, cnt + 0);
    if (sd >= 0 && sd < p.k_sel) direct[sd] = j;
    const int sc = warp_append(is_cand, cnt + 1);
    if (sc >= 0 && sc < p.kv.max_len) {
      ct[sc] = t;
      cj[sc] = j;
    }
  }
}

// ----------------------------------------------------------------------------
// 3. finish: exact select + float64 refinement + window merge + sort
// ----------------------------------------------------------------------------
constexpr int kFinThreads = 1024;

// Radix select over the elements e in [0, n) with pred(e): the r-th largest
// (1-based) of key(e), a KeyT of KBITS bits, 8 bits per pass.  Returns the key;
// *n_gt receives how many selected elements are strictly greater.
template <typename KeyT, int KBITS, typename KeyFn, typename PredFn>
__device__ KeyT block_kth_largest(int n, int r, KeyFn key, PredFn pred, uint32_t* n_gt) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t sh_digit, sh_rem;
  KeyT prefix = 0, mask = 0;
  uint32_t rem = (uint32_t)r, gt = 0;
  for (int shift = KBITS - 8; shift >= 0; shift -= 8) {
    for (int e = threadIdx.x; e < 256; e += blockDim.x) hist[e] = 0u;
    __syncthreads();
    for (int e = threadIdx.x; e < n; e += blockDim.x) {
      if (!pred(e)) continue;
      const KeyT k = key(e);
      if ((k & mask) == prefix) atomicAdd(&hist[(uint32_t)(k >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      uint32_t cum = 0;
      int dg = 255;
      for (; dg > 0; --dg) {
        if (cum + hist[dg] >= rem) break;
        cum += hist[dg];
      }
      sh_digit = (uint32_t)dg;
      sh_rem = rem - cum;
      gt += cum;
    }
    __syncthreads();
    prefix |= (KeyT)sh_digit << shift;
    mask |= (KeyT)255 << shift;
    rem = sh_rem;
    __syncthreads();
  }
  if (threadIdx.x == 0) *n_gt = gt;  // greater-count accumulated by thread 0 only
  __syncthreads();
  return prefix;
}

template <int H, bool FP8>
__global__ void __launch_bounds__(kFinThreads) select_finish_kernel(SelectParams p) {
  __shared__ int sel[kMaxIdxWidth];
  __shared__ uint32_t n_sel, n_band_s, gt_s;
  __shared__ double dlt[H];
  const int bq = blockIdx.x;
  const int b = bq / p.n_q, i = bq % p.n_q;
  const int L = seq_len(p.kv, b, p.n_q, p.status, false);
  const int pos = L - p.n_q + i;
  const int width = p.window + p.k_sel;
  const int n_c = pos - p.window + 1;
  int32_t* out = p.idx + (size_t)bq * width;
  if (n_c <= p.k_sel) {
    for (int e = threadIdx.x; e < width; e += blockDim.x) out[e] = e <= pos ? e : -1;
    return;
  }
  const uint32_t* cnt = p.counters + (size_t)bq * 8;
  const uint32_t n_direct = min(__ldcg(cnt + 0), (uint32_t)p.k_sel);
  const uint32_t n_cand = min(__ldcg(cnt + 1), (uint32_t)p.kv.max_len);
  const float eps = __uint_as_float(__ldcg(p.selmeta + (size_t)bq * 4 + 1));
  const int need = p.k_sel - (int)n_direct;  // >= 1 by construction
  const float* ct = p.cand_t + (size_t)bq * p.kv.max_len;
  const int32_t* cj = p.cand_j + (size_t)bq * p.kv.max_len;
  if (threadIdx.x == 0) {
    n_sel = 0;
    n_band_s = 0;
  }
  __syncthreads();

  // tau: the need-th largest float32 key among the candidates.
  const uint32_t tau_key = block_kth_largest<uint32_t, 32>(
      (int)n_cand, need, [&](int e) { return ordered_key(__ldcg(ct + e)); },
      [](int) { return true; }, &gt_s);
  const float tau = key_to_float(tau_key);
  const float hi_b = tau + eps, lo_b = tau - eps;

  // Kept outright: the direct list and candidates above the band.  Band -> refine.
  auto push = [&](int j) {
    const uint32_t slot = atomicAdd(&n_sel, 1u);
    if (slot < (uint32_t)kMaxIdxWidth) sel[slot] = j;
  };
  for (uint32_t e = threadIdx.x; e < n_direct; e += blockDim.x)
    push(__ldcg(p.direct + (size_t)bq * p.k_sel + e));
  int32_t* bj = p.band_j + (size_t)bq * p.kv.max_len;
  double* bt = p.band_t + (size_t)bq * p.kv.max_len;
  for (uint32_t e = threadIdx.x; e < n_cand; e += blockDim.x) {
    const float t = __ldcg(ct + e);
    if (t > hi_b) push(__ldcg(cj + e));
    else if (t >= lo_b) bj[atomicAdd(&n_band_s, 1u)] = __ldcg(cj + e);
  }
  for (int hd = threadIdx.x; hd < H; hd += blockDim.x) dlt[hd] = p.delta64[(size_t)bq * H + hd];
  __syncthreads();
  const int n_band = (int)n_band_s;
  const int need2 = p.k_sel - (int)n_sel;  // taken from the band

  if (need2 > 0) {
    // float64 re-scoring of the band: one warp per key, lanes split the dimension.
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const double scale = (double)p.sm_scale;
    for (int e = warp; e < n_band; e += blockDim.x / 32) {
      const int j = bj[e];
      const size_t row = (size_t)b * p.kv.max_len + j;
      double kx[4];
      if (FP8) {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(
            static_cast<const uint8_t*>(p.kv.k) + row * kHeadDim + lane * 4);
        const double ks = (double)p.kv.k_scale[row];
#pragma unroll
        for (int t = 0; t < 4; ++t) kx[t] = e4m3_to_f64((w >> (8 * t)) & 0xffu) * ks;
      } else {
        const uint2 w = *reinterpret_cast<const uint2*>(
            static_cast<const uint16_t*>(p.kv.k) + row * kHeadDim + lane * 4);
        kx[0] = bf16_bits_to_f32(w.x & 0xffffu);
        kx[1] = bf16_bits_to_f32(w.x >> 16);
        kx[2] = bf16_bits_to_f32(w.y & 0xffffu);
        kx[3] = bf16_bits_to_f32(w.y >> 16);
      }
      double best = -INFINITY;
      for (int hd = 0; hd < H; ++hd) {
        const uint2 qw = __ldg(reinterpret_cast<const uint2*>(
            p.q + ((size_t)bq * H + hd) * kHeadDim + lane * 4));
        double d = (double)bf16_bits_to_f32(qw.x & 0xffffu) * kx[0] +
                   (double)bf16_bits_to_f32(qw.x >> 16) * kx[1] +
                   (double)bf16_bits_to_f32(qw.y & 0xffffu) * kx[2] +
                   (double)bf16_bits_to_f32(qw.y >> 16) * kx[3];
        d = warp_sum_d(d);
        best = fmax(best, scale * d - dlt[hd]);
      }
      if (lane == 0) bt[e] = best;
    }
    __threadfence_block();
    __syncthreads();
    // Boundary value among the band, then the lowest positions among its ties.
    const unsigned long long vb = block_kth_largest<unsigned long long, 64>(
        n_band, need2, [&](int e) { return ordered_key64(bt[e]); }, [](int) { return true; },
        &gt_s);
    const uint32_t n_gt = gt_s;
    const int take_eq = need2 - (int)n_gt;
    const uint32_t jb_inv = block_kth_largest<uint32_t, 32>(
        n_band, take_eq, [&](int e) { return ~(uint32_t)bj[e]; },
        [&](int e) { return ordered_key64(bt[e]) == vb; }, &gt_s);
    const int jb = (int)~jb_inv;
    for (int e = threadIdx.x; e < n_band; e += blockDim.x) {
      const unsigned long long kk = ordered_key64(bt[e]);
      if (kk > vb || (kk == vb && bj[e] <= jb)) push(bj[e]);
    }
  }
  // The forced recent window [p - window + 1, p].
  for (int j = n_c + threadIdx.x; j <= pos; j += blockDim.x) push(j);
  __syncthreads();
  // Bitonic sort of the selection (ascending), padded to a power of two.
  const int n = (int)min(n_sel, (uint32_t)kMaxIdxWidth);
  int np2 = 1;
  while (np2 < n) np2 <<= 1;
  for (int e = n + threadIdx.x; e < np2; e += blockDim.x) sel[e] = 0x7fffffff;
  __syncthreads();
  for (int kk = 2; kk <= np2; kk <<= 1) {
    for (int jj = kk >> 1; jj > 0; jj >>= 1) {
      for (int e = threadIdx.x; e < np2; e += blockDim.x) {
        const int partner = e ^ jj;
        if (partner > e) {
          const bool up = (e & kk) == 0;
          const int a = sel[e], c = sel[partner];
          if ((a > c) == up) {
            sel[e] = c;
            sel[partner] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int e = threadIdx.x; e < width; e += blockDim.x) out[e] = e < n ? sel[e] : -1;
}

// ----------------------------------------------------------------------------
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
  importance_simt_kernel<H, FP8><<<dim3(p.splits2, bq), kThreads, smem, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  select_compact_kernel<<<dim3(p.splits3, bq), kThreads, 0, st>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  select_finish_kernel<H, FP8><<<bq, kFinThreads, 0, st>>>(p);
  return cudaGetLastError();
}

template <int H, bool FP8>
static cudaError_t launch_rest_t(const SelectParams& p, int batch, cudaStream_t st) {
  const int bq = batch * p.n_q;
  select_compact_kernel<<<dim3(p.splits3, bq), kThreads, 0, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  select_finish_kernel<H, FP8><<<bq, kFinThreads, 0, st>>>(p);
  return cudaGetLastError();
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
