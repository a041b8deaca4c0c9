// Fused tail of the one-token full layer: after streaming their key chunks, the CTAs
// of one (sequence, token) row merge their split partials and select the row's tokens
// together, so that the step needs no separate merge, importance or selection kernels.
//
// The selection (web coverage of HySparse2: toolnavs article 2080, fr "Ce que fait
// HySparse2", paragraph on selection granularity -- the last `window` positions, plus
// the top `k_sel` positions outside the window ranked by the full layer's own scores)
// ranks key j by t_j = max_h (x_hj - D_h), x_hj = s_hj log2(e) its logit in log2 units
// and D_h = lse2_h - min_h' lse2_h' (log2 units): the same order as max_h exp(s_hj -
// lse_h).  The lse is only known once every chunk of the row is done, so during the
// stream each key records only the bound
//     u_j = max_h x_hj,     u_j - W <= t_j <= u_j,     W = max_h D_h,
// and counts u_j in a shared-memory histogram, linear in u.  Then, per row (CTA r of the
// row owns the positions [r chunk, (r + 1) chunk) for the selection, whichever CTA
// streamed them):
//   1. every CTA publishes its m per head and its histogram and arrives at the row's first
//      barrier, then copies its chunk's bounds and the row's histogram on chip and computes
//      the row's lse from the split partials;
//   2. the bin holding the k_sel-th largest u gives a lower edge lo; no key with
//      u_j < lo - W - 2 eps can be among the top k_sel (the k_sel-th largest t, T, is at
//      least lo - W), so only the other keys of its chunk -- the candidates, a few per
//      thousand -- get their exact float32 t_j, from their K rows gathered again through
//      the tensor cores.  Each CTA keeps its candidates (ascending positions) and counts
//      them in the row's fine histogram of t over [lo - W - 2 eps, hi], which holds T;
//   3. after the second barrier the fine histogram gives the bin B of the k_sel-th
//      largest t; with m bins of width at least eps around it, keys of bins >= B + m are
//      in, keys of bins < B - m are out.  Each CTA counts its own keys that are in, and
//      re-scores its own keys of the band between in float64 into the row's band list;
//   4. after the third barrier every CTA ranks the band by (key desc, position asc) and
//      writes the selected positions of its own chunk, in order, from the slot after those
//      of the lower chunks (their counts, and the band keys below its chunk that the
//      ranking takes); the first CTA appends the window.  Then the CTA lets the next
//      kernel start.  (Each CTA merges its share of the row's output between arriving at
//      the second barrier and waiting there.)
// The float32 keys are within eps / 2 of the exact ones, eps = 1e-3 max(1, |bin edge| +
// W) (as in the separate selection kernels), so the chosen set is the float64
// definition's up to the tie band.
//
// The CTAs of a row wait for one another at the barriers: the kernel is launched
// cooperatively (all CTAs resident) whenever a row has more than one CTA, and every
// wait gives up after a bounded number of cycles, recording HS2_ERR_DEVICE_TIMEOUT.
#pragma once

#include "hs2_internal.cuh"
#include "select_common.cuh"
#include "sm100.cuh"

namespace hs2 {

constexpr int kUBins = 2048;         // bins of the u histogram and of the fine t histogram
constexpr float kUScale = 16.f;      // u bins per log2 unit
constexpr float kUOrigin = -64.f;    // lower edge of u bin 1 is kUOrigin + 1/16
constexpr float kSelEps = 1e-3f;
constexpr long long kRowSpinCycles = 4000000000ll;
constexpr int kBandSmem = 512;       // bands up to this size are ranked pairwise on chip
constexpr int kTailTiles = 2;        // candidate tiles (128 keys) gathered at a time
static_assert(2 * kUBins <= kHistBins, "the u and fine histograms share a row's histogram region");

// Slots of a row's synchronisation words (the first two belong to the separate selection
// kernels).
enum : int { kRowNBand = 2, kRowArrive1 = 3, kRowArrive2 = 4, kRowArrive3 = 5, kRowDone = 6 };

// Histogram bin of a bound u: monotone in u, u below -64 + 1/16 in bin 0 and u at or above
// 64 - 1/16 in the last bin (a NaN goes to bin 0).
__device__ __forceinline__ int ubin(float u) {
  float y = (u - kUOrigin) * kUScale;
  y = fminf(fmaxf(y, 0.f), (float)(kUBins - 1));
  return (int)y;
}
// Nominal lower edge of bin b.
__device__ __forceinline__ float ubin_edge(int b) { return (float)b / kUScale + kUOrigin; }
// A value at or below every u whose bin is b or higher: the edge less the rounding of
// u - kUOrigin (at most 2^-18 below 128) and of this subtraction.
__device__ __forceinline__ float ubin_floor(int b) {
  return b <= 0 ? -INFINITY : ubin_edge(b) - 3e-5f;
}

// The fine histogram of t over [lo, lo + kUBins / inv_w): monotone, clamped at both ends.
struct FineBins {
  float lo, inv_w;
  __device__ __forceinline__ int bin(float t) const {
    float y = (t - lo) * inv_w;
    y = fminf(fmaxf(y, 0.f), (float)(kUBins - 1));
    return (int)y;
  }
};

// Shared-memory histograms are dense (bin b at word b), as in global memory, so that one
// bulk reduction publishes a CTA's histogram and 16-byte copies bring the row's back.
constexpr uint32_t kUHistBytes = kUBins * 4u;

// ---- row barriers: every CTA of a row arrives once per counter and call, then waits
// until `target` have.  Arrival: a block barrier, then a release reduction by thread 0
// (the CTA's earlier writes, ordered by the block barrier, become visible to whoever
// acquires the counter).  Waiting: thread 0 spins on an acquire load (a bounded number of
// cycles), then a block barrier.
__device__ __forceinline__ void row_arrive(uint32_t* counter) {
  __syncthreads();
  if (threadIdx.x == 0) sm100::red_release_gpu_add(counter, 1u);
}
// `stall` (the stall test) waits for one CTA more than the row has, with a short limit.
static __device__ __noinline__ bool row_wait(uint32_t* counter, uint32_t target, bool stall) {
  __shared__ uint32_t ok_s;
  if (threadIdx.x == 0) {
    uint32_t ok = 1;
    const long long limit = stall ? kStallTestCycles : kRowSpinCycles;
    target += stall ? 1u : 0u;
    if (sm100::ld_acquire_gpu_u32(counter) < target) {
      const long long t0 = clock64();
      while (sm100::ld_acquire_gpu_u32(counter) < target) {
        if (clock64() - t0 > limit) {
          ok = 0;
          break;
        }
        __nanosleep(100);  // leave the counter's L2 slice to the others
      }
    }
    ok_s = ok;
  }
  __syncthreads();
  return ok_s != 0;
}

// The bin B holding the k-th largest element of a dense shared-memory histogram (0 if
// there are fewer than k), and with mb > 0 the counts in the bins >= B + mb (`above`)
// and in [B - mb, B + mb) (`near`).  Threads t < 128 own the bins [kUBins - 16(t + 1),
// kUBins - 16 t) (thread 0 the top ones), read as four 16-byte chunks starting at chunk
// t mod 4 so that a warp's loads meet at most 4-way bank conflicts; one block-wide scan
// from the top finds the owner of the k-th element, which walks its 16 bins.  Every
// thread calls it (blockDim >= 128) and gets the result.  The tail runs this code once
// per launch and histogram, so it is one out-of-line copy.
struct BinScan {
  int bin;
  uint32_t above, near;
};
static __device__ __noinline__ BinScan scan_bins(const uint32_t* hs, int k, int mb) {
  static_assert(kUBins == 128 * 16, "16 bins per scanning thread");
  __shared__ uint32_t wtot[4];
  __shared__ uint32_t wsum2[2][4];
  __shared__ BinScan out_s;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool own = tid < 128;
  const int base = kUBins - 16 * (tid + 1);
  uint32_t v[16];  // v[4c + q]: bin base + 4c + q
  uint32_t sum = 0;
  if (own) {
    const uint4* row = reinterpret_cast<const uint4*>(hs + base);
    uint4 c[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) c[u] = row[(u + tid) & 3];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int ch = (u + tid) & 3;
#pragma unroll
      for (int ch2 = 0; ch2 < 4; ++ch2)
        if (ch == ch2) {
          v[4 * ch2] = c[u].x;
          v[4 * ch2 + 1] = c[u].y;
          v[4 * ch2 + 2] = c[u].z;
          v[4 * ch2 + 3] = c[u].w;
        }
    }
#pragma unroll
    for (int e = 0; e < 16; ++e) sum += v[e];
  } else {
#pragma unroll
    for (int e = 0; e < 16; ++e) v[e] = 0u;
  }
  uint32_t incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  if (own && lane == 31) wtot[warp] = incl;
  if (tid == 0) out_s.bin = 0;
  __syncthreads();
  uint32_t before = incl - sum;  // in the bins above this thread's
  for (int w = 0; w < warp && w < 4; ++w) before += wtot[w];
  if (own && before < (uint32_t)k && (uint32_t)k <= before + sum) {
    uint32_t cum = before;
    int bin = base;
#pragma unroll
    for (int e = 15; e >= 0; --e) {
      cum += v[e];
      if (cum >= (uint32_t)k) {
        bin = base + e;
        break;
      }
    }
    out_s.bin = bin;
  }
  __syncthreads();
  BinScan r;
  r.bin = out_s.bin;
  r.above = 0u;
  r.near = 0u;
  if (mb > 0) {
    const int B = r.bin;
    uint32_t above = 0, near = 0;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int bb = base + e;
      above += bb >= B + mb ? v[e] : 0u;
      near += (bb >= B - mb && bb < B + mb) ? v[e] : 0u;
    }
    above = __reduce_add_sync(0xffffffffu, above);
    near = __reduce_add_sync(0xffffffffu, near);
    if (own && lane == 0) {
      wsum2[0][warp] = above;
      wsum2[1][warp] = near;
    }
    __syncthreads();
    r.above = (wsum2[0][0] + wsum2[0][1]) + (wsum2[0][2] + wsum2[0][3]);
    r.near = (wsum2[1][0] + wsum2[1][1]) + (wsum2[1][2] + wsum2[1][3]);
    __syncthreads();  // wsum2 and out_s are reused by the next call
  } else {
    __syncthreads();
  }
  return r;
}

// Asynchronous copies (cp.async, waited for with cp_async_wait_all) by all threads:
// a global histogram into a dense shared-memory copy, and n 4-byte words.
__device__ __forceinline__ void async_bins(uint32_t* hs, const uint32_t* gh) {
  for (int v = threadIdx.x; v < kUBins / 4; v += blockDim.x)
    sm100::cp_async_16(sm100::smem_u32(hs + 4 * v), gh + 4 * v, 16u);
}
__device__ __forceinline__ void async_words(void* dst, const void* src, int n) {
  const int nv = (n + 3) / 4;
  for (int v = threadIdx.x; v < nv; v += blockDim.x) {
    const int left = n - 4 * v;
    sm100::cp_async_16(sm100::smem_u32(static_cast<uint8_t*>(dst) + 16 * v),
                       static_cast<const uint8_t*>(src) + 16 * v, left >= 4 ? 16u : 4u * left);
  }
}

// Block-wide ordered compaction: the indices e of [0, m) with pred(e), in increasing
// order, each handed to emit(rank, e); returns the count to every thread.  Each thread takes a
// contiguous run of up to 64 indices (independent loads, a bit mask), then one block-wide
// exclusive scan of the counts places the runs: no atomics on a shared counter, whose
// round trips would serialise a loop run by a handful of warps.  All threads call.
template <typename Pred, typename Emit>
__device__ __forceinline__ int block_compact(int m, Pred pred, Emit emit) {
  __shared__ uint32_t wsum[32];
  const int nt = blockDim.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nw = nt >> 5;
  int total = 0;
  for (int c0 = 0; c0 < m; c0 += 64 * nt) {
    const int cm = min(64 * nt, m - c0);
    const int R = (cm + nt - 1) / nt;
    const int e0 = c0 + tid * R, e1 = min(e0 + R, c0 + cm);
    unsigned long long mask = 0ull;
#pragma unroll 8
    for (int e = e0; e < e1; ++e)
      if (pred(e)) mask |= 1ull << (e - e0);
    const uint32_t cnt = (uint32_t)__popcll(mask);
    uint32_t incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += x;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    uint32_t before = 0, all = 0;
    for (int w = 0; w < nw; ++w) {
      const uint32_t c = wsum[w];
      before += w < warp ? c : 0u;
      all += c;
    }
    uint32_t at = (uint32_t)total + before + incl - cnt;
    while (mask) {
      const int r = __ffsll(mask) - 1;
      mask &= mask - 1;
      emit((int)at++, e0 + r);
    }
    total += (int)all;
    __syncthreads();  // wsum is reused by the next chunk or call
  }
  return total;
}

// The row's log-sum-exp per head, from its split partials.
template <int H>
struct RowLse {
  float M[H];      // largest m over the non-empty splits (log2 units)
  float invL[H];   // 1 / sum_s l_s 2^(m_s - M)
  double lse2[H];  // M + log2 sum_s l_s 2^(m_s - M)  (log2 units)
  double dl[H];    // (lse2 - min_h lse2) ln 2: the float64 shifts of the re-scoring
  float D[H];      // lse2 - min_h lse2 (log2 units, float32)
  float W;         // max_h D
};

// Ordered 32-bit keys of float32 values for an unsigned atomicMax (key 0, the zero state,
// is below every value).
__device__ __forceinline__ uint32_t max_key(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float max_key_value(uint32_t k) {
  return k == 0u ? -INFINITY : __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Every thread calls this; pml: the row's partials [S][H][2] (m in log2 units, l); rowmax:
// the ordered keys of the row's largest m per head (every CTA of the row adds its own
// before the first barrier); tmp: blockDim.x float2 of shared scratch.  M_h is that
// largest m, and L_h = sum_s l_s 2^(m_s - M_h), each weight in float32 (relative error
// below 2^-22, well under that of the partial sums l) summed without loss (two-sum).
// Thread t takes head t % H and the splits t / H, t / H + G, ... (G = blockDim / H), so
// consecutive threads read consecutive partials.  log2 L is taken on the mantissa of its
// leading float (log2f of a value in [0.5, 1), absolute error about 2^-24) plus the
// exponent and the first-order term of the trailing float, and assembled with M in
// float64: lse2 carries about 2^-23 absolute, well inside the 1e-6 tie band of the
// selection.  The shifts D and dl are taken from C, a common value just below the
// smallest lse2 (the ranking does not depend on which).  Every CTA of the row reads the
// same partials in the same order, so all get the same bits.
template <int H>
static __device__ __noinline__ void row_lse(const float* __restrict__ pml,
                                            const uint32_t* __restrict__ rowmax, int S,
                                            RowLse<H>& r, float2* tmp) {
  const int nt = blockDim.x, tid = threadIdx.x, lane = tid & 31;
  const int G = nt / H;
  const int h = tid % H, g = tid / H;
  // The thread's first kFirst partials are requested with the maxima (one round trip).
  constexpr int kFirst = 4;
  const float2* src = reinterpret_cast<const float2*>(pml) + h;
  float2 first[kFirst];
#pragma unroll
  for (int k = 0; k < kFirst; ++k) {
    const int s = g + k * G;
    first[k] = g < G && s < S ? __ldcg(src + (size_t)s * H) : make_float2(0.f, 0.f);
  }
  if (tid < H) r.M[tid] = max_key_value(__ldcg(rowmax + tid));
  __syncthreads();
  float ls = 0.f, le = 0.f;
  if (g < G) {
    const float M = r.M[h];
#pragma unroll
    for (int k = 0; k < kFirst; ++k)
      if (first[k].y > 0.f) two_sum_acc(ls, le, first[k].y * exp2f(first[k].x - M));
#pragma unroll 8
    for (int s = g + kFirst * G; s < S; s += G) {
      const float2 v = __ldcg(src + (size_t)s * H);
      if (v.y > 0.f) two_sum_acc(ls, le, v.y * exp2f(v.x - M));
    }
  }
  tmp[tid] = make_float2(ls, le);
  __syncthreads();
  if (tid < H) {
    ls = 0.f;
    le = 0.f;
#pragma unroll 1
    for (int g2 = 0; g2 < G; ++g2) {
      const float2 v = tmp[g2 * H + tid];
      le += v.y;
      two_sum_acc(ls, le, v.x);
    }
    const float lh = ls + le;         // leading float of L
    const float ll = (ls - lh) + le;  // and the rest
    if (lh > 0.f) {
      int ex;
      const float mant = frexpf(lh, &ex);  // lh = mant 2^ex, mant in [0.5, 1)
      r.invL[tid] = 1.f / lh;
      r.lse2[tid] = (double)r.M[tid] + (double)ex + (double)log2f(mant) +
                    (double)(ll / lh * 1.4426950408889634f);
    } else {
      r.invL[tid] = 0.f;
      r.lse2[tid] = -INFINITY;
    }
  }
  __syncthreads();
  if (tid < 32) {
    float mn = INFINITY;
#pragma unroll 1
    for (int hh = lane; hh < H; hh += 32) mn = fminf(mn, (float)r.lse2[hh]);
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 16));
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 8));
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 4));
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 2));
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 1));
    const double c = (double)mn - 1e-5 * fmax(1.0, fabs((double)mn));  // at or below every lse2
    float w = 0.f;
#pragma unroll 1
    for (int hh = lane; hh < H; hh += 32) {
      const double d = r.lse2[hh] - c;
      r.D[hh] = (float)d;
      r.dl[hh] = d * 0.69314718055994530942;
      w = fmaxf(w, (float)d);
    }
    w = fmaxf(w, __shfl_xor_sync(0xffffffffu, w, 16));
    w = fmaxf(w, __shfl_xor_sync(0xffffffffu, w, 8));
    w = fmaxf(w, __shfl_xor_sync(0xffffffffu, w, 4));
    w = fmaxf(w, __shfl_xor_sync(0xffffffffu, w, 2));
    w = fmaxf(w, __shfl_xor_sync(0xffffffffu, w, 1));
    if (lane == 0) r.W = w * (1.f + 1e-6f);  // covers the rounding of D to float
  }
  __syncthreads();
}

// The outputs (h, d) of a row that CTA r merges: [r P, (r + 1) P) with P = ceil(H
// kHeadDim / S) rounded up to a multiple of 4 (so that each split's part of the share is
// a 16-byte-aligned run); MergeShare also gives the heads the share spans.
struct MergeShare {
  int o0, o1, opc;
  int h0, nh;  // heads [h0, h0 + nh), h0 even and nh even: whole 16-byte (m, l) pairs
};
template <int H>
__device__ __forceinline__ MergeShare merge_share(int split, int S) {
  constexpr int kOut = H * kHeadDim;
  MergeShare m;
  m.opc = (((kOut + S - 1) / S) + 3) & ~3;
  m.o0 = min(split * m.opc, kOut);
  m.o1 = min(m.o0 + m.opc, kOut);
  m.h0 = (m.o0 / kHeadDim) & ~1;
  m.nh = m.o1 > m.o0 ? (((m.o1 - 1) / kHeadDim + 2) & ~1) - m.h0 : 0;
  return m;
}

// Bytes of shared memory that prefetch_merge fills (a multiple of 16).
template <int H>
__device__ __forceinline__ uint32_t merge_prefetch_bytes(int split, int S) {
  const MergeShare m = merge_share<H>(split, S);
  return (uint32_t)S * m.opc * 4u + (uint32_t)S * m.nh * 8u;
}

// The split partials this CTA's share of the merge reads, copied on chip (cp.async, all
// threads): o of every split for the share's outputs ([S][opc] floats at mo), then (m, l)
// of every split for the share's heads ([S][nh] float2 after it).
template <int H>
__device__ __forceinline__ void prefetch_merge(const FullParams& p, int bq, int split, int S,
                                               float* mo) {
  const MergeShare m = merge_share<H>(split, S);
  const float* po = p.part_o + (size_t)bq * S * H * kHeadDim;
  const float* pml = p.part_ml + (size_t)bq * S * H * 2;
  const int n4 = (m.o1 - m.o0) / 4;  // 16-byte chunks of one split
  for (int e = threadIdx.x; e < S * n4; e += blockDim.x) {
    const int s = e / n4, c = e % n4;
    sm100::cp_async_16(sm100::smem_u32(mo + s * m.opc + 4 * c),
                       po + (size_t)s * H * kHeadDim + m.o0 + 4 * c, 16u);
  }
  float* ml = mo + S * m.opc;
  const int n2 = m.nh / 2;  // 16-byte chunks (two heads) of one split
  for (int e = threadIdx.x; e < S * n2; e += blockDim.x) {
    const int s = e / n2, c = e % n2;
    sm100::cp_async_16(sm100::smem_u32(ml + 4 * e), pml + ((size_t)s * H + m.h0 + 2 * c) * 2, 16u);
  }
}

// This CTA's share of the row's merged output, out_h = sum_s 2^(m_s - M) o_s / L: each
// output is summed by G = blockDim / P threads over every G-th split (consecutive
// threads take consecutive outputs of one split), and the G sums meet in shared memory
// (tmp: blockDim.x floats).  The partials come from `mo` (prefetch_merge, complete) or,
// if null, from global memory.  The thread holding d = 0 of a head writes its lse
// (natural log) to lse64 and lse_out.  Every thread calls it.
template <int H>
static __device__ __noinline__ void row_merge(const FullParams& p, int bq, int split, int S,
                                              const RowLse<H>& r, float* tmp, const float* mo) {
  const float* po = p.part_o + (size_t)bq * S * H * kHeadDim;
  const float2* pml = reinterpret_cast<const float2*>(p.part_ml + (size_t)bq * S * H * 2);
  constexpr int kOut = H * kHeadDim;
  const MergeShare m = merge_share<H>(split, S);
  const float2* mml = reinterpret_cast<const float2*>(mo + S * m.opc);
  const int nt = blockDim.x, tid = threadIdx.x;
  const int P = min(m.opc, nt);  // outputs per round
  const int G = nt / P;          // threads per output
  const int ol = tid % P, g = tid / P;
#pragma unroll 1
  for (int ob = m.o0; ob < m.o1; ob += P) {
    const int o = ob + ol;
    const bool mine = g < G && o < m.o1;
    const int h = o / kHeadDim, d = o % kHeadDim;
    float acc = 0.f;
    if (mine) {
      const float M = r.M[h], il = r.invL[h];
      if (mo) {
#pragma unroll 4
        for (int s = g; s < S; s += G) {
          const float2 ml = mml[s * m.nh + h - m.h0];
          if (ml.y > 0.f) acc = fmaf(exp2f(ml.x - M) * il, mo[s * m.opc + o - m.o0], acc);
        }
      } else {
#pragma unroll 16
        for (int s = g; s < S; s += G) {
          const float2 ml = __ldcg(pml + (size_t)s * H + h);
          const float v = __ldcg(po + ((size_t)s * H + h) * kHeadDim + d);
          if (ml.y > 0.f) acc = fmaf(exp2f(ml.x - M) * il, v, acc);
        }
      }
    }
    if (G > 1) {
      tmp[tid] = acc;
      __syncthreads();
      if (mine && g == 0)
#pragma unroll 1
        for (int g2 = 1; g2 < G; ++g2) acc += tmp[g2 * P + ol];
      __syncthreads();
    }
    if (mine && g == 0) {
      p.out[(size_t)bq * kOut + o] = acc;
      if (d == 0) {
        const double lse = r.lse2[h] * 0.69314718055994530942;
        if (p.lse64) p.lse64[(size_t)bq * H + h] = lse;
        if (p.lse_out) p.lse_out[(size_t)bq * H + h] = (float)lse;
      }
    }
  }
}

// Index row of a row that keeps every position (no more than k_sel positions outside the
// window): [0, pos], then -1.
__device__ __forceinline__ void write_all_positions(int32_t* out_row, int width, int pos) {
  for (int e = threadIdx.x; e < width; e += blockDim.x) out_row[e] = e <= pos ? e : -1;
}

// Where the tail finds the query for the float64 re-scoring (byte strides of heads and of
// 8-element chunks, as rescore_f64 takes them).
struct QView {
  const uint8_t* base;
  int hstride, cstride;
};

// Position of j in a CTA's ascending list of candidate positions oj[0, n) (an entry may
// hold ~j once taken: the order of the plain values is kept).
__device__ __forceinline__ int find_position(const int* oj, int n, int j) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    const int v = oj[mid];
    if ((v < 0 ? ~v : v) < j) lo = mid + 1;
    else hi = mid;
  }
  return lo;
}

// Steps 2 to 4 of the selection (see the top of this file), after the row's first barrier
// and lse, with this CTA's first `piece` bounds already in `us`.  All threads of every CTA
// of the row call it.  `recompute(list, m, t2, round, D)` (all threads) gathers the K rows
// of the positions list[0, m) (m <= kTailTiles * 128), runs them through the stream's S =
// K Q^T MMA and stores t = max_h (x_h - D[h]) of each into t2[0, m), ending with a block
// barrier; it returns false if a wait gave up.  `scratch` (the gathered tiles' space) is
// free once the candidates are re-scored.  Returns false if a wait gave up.
template <int H, bool FP8, typename Recompute, typename Merge>
__device__ __forceinline__ bool row_select(const FullParams& p, uint8_t* scratch, float* us,
                                           int* cl, float* t2s, int piece, int bq, int b,
                                           int split, int S, int k0, int c_hi, int n_c, int pos,
                                           int bk, const RowLse<H>& rl, const QView& qv,
                                           Recompute&& recompute, Merge&& merge) {
  __shared__ float eps_s;
  __shared__ FineBins fb_s;
  __shared__ int mb_s;
  __shared__ uint32_t red_s[2][32];
  const int nt = blockDim.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = nt >> 5;
  const int width = p.window + p.k_sel;
  int32_t* out_row = p.sel_idx + (size_t)bq * width;
  const size_t rowoff = (size_t)bq * p.kv.max_len;
  uint32_t* rs = p.rowsync + (size_t)bq * 8;
  uint32_t* gfh = p.uhist + (size_t)bq * kHistBins + kUBins;  // the row's fine histogram
  uint32_t* rowcnt = p.rowcnt + (size_t)bq * kSmCountBound;
  bool ok = true;

  // Block-wide sums of two counters (all threads call; the result to every thread).
  auto block_sum2 = [&](uint32_t& x, uint32_t& y) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      x += __shfl_xor_sync(0xffffffffu, x, o);
      y += __shfl_xor_sync(0xffffffffu, y, o);
    }
    if (lane == 0) {
      red_s[0][warp] = x;
      red_s[1][warp] = y;
    }
    __syncthreads();
    x = 0u;
    y = 0u;
    for (int w = 0; w < nwarps; ++w) {
      x += red_s[0][w];
      y += red_s[1][w];
    }
    __syncthreads();
  };

  if (tid == 0) {
    const float edge = fmaxf(fabsf(ubin_edge(bk)), fabsf(ubin_edge(bk + 1)));
    const float eps = kSelEps * fmaxf(1.f, edge + rl.W);
    // T (the k_sel-th largest t) lies in [floor(bk) - W, edge(bk + 1)]: the fine bins
    // span that with a margin; keys outside fall into the end bins.
    const float lo = bk <= 0 ? kUOrigin - 64.f - rl.W : ubin_floor(bk) - rl.W - 2.f * eps;
    const float hi = bk >= kUBins - 1 ? lo + 2.f * rl.W + 64.f : ubin_edge(bk + 1) + 3e-5f;
    FineBins fb;
    fb.lo = lo;
    fb.inv_w = (float)kUBins / fmaxf(hi - lo, 1e-6f);
    fb_s = fb;
    eps_s = eps;
    // mb bins of the fine histogram cover eps, with a spare bin for rounding.
    mb_s = (int)ceilf(eps * fb.inv_w) + 2;
  }
  __syncthreads();
  const float eps = eps_s;
  const FineBins fb = fb_s;
  const int mb = mb_s;
  const float theta = ubin_floor(bk) - rl.W - 2.f * eps;

  // ---- 2. this chunk's candidates, a piece at a time, through the tensor cores in rounds
  // of kTailTiles tiles.  Their keys go to the row's fine histogram and to this CTA's list
  // (ascending positions): on chip when the chunk is one piece, else in the row's
  // candidate rows at the chunk's offset.
  const bool one_piece = c_hi - k0 <= piece;
  float* ot = one_piece ? us : p.cand_t + (size_t)bq * p.ld_u + k0;
  int* oj = one_piece ? cl : p.cand_j + (size_t)bq * p.ld_u + k0;
  int own_n = 0;
  uint32_t round = 0;
  for (int pc = k0; pc < c_hi; pc += piece) {
    const int m = min(piece, c_hi - pc);
    if (pc != k0) {  // later pieces (long chunks only) are staged here
      __syncthreads();
      async_words(us, p.ubuf + (size_t)bq * p.ld_u + pc, m);
      sm100::cp_async_wait_all();
    }
    __syncthreads();
    const int ncl = block_compact(
        m, [&](int e) { return us[e] >= theta; }, [&](int at, int e) { cl[at] = pc + e; });
    for (int r0 = 0; r0 < ncl; r0 += kTailTiles * 128, ++round) {
      const int mm = min(kTailTiles * 128, ncl - r0);
      if (!recompute(cl + r0, mm, t2s, round, rl.D)) ok = false;
      uint32_t top = 0, bot = 0;
      for (int e = tid; e < mm; e += nt) {
        const float t = t2s[e];
        const int bb = fb.bin(t);
        if (bb == kUBins - 1) ++top;
        else if (bb == 0) ++bot;
        else atomicAdd(gfh + bb, 1u);
        if (one_piece) {
          us[r0 + e] = t;  // the bounds were consumed by the compaction
        } else {
          ot[own_n + r0 + e] = t;
          oj[own_n + r0 + e] = cl[r0 + e];
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        top += __shfl_xor_sync(0xffffffffu, top, o);
        bot += __shfl_xor_sync(0xffffffffu, bot, o);
      }
      if (lane == 0) {
        if (top) atomicAdd(gfh + kUBins - 1, top);
        if (bot) atomicAdd(gfh, bot);
      }
      __syncthreads();  // t2s is refilled by the next round
    }
    own_n += ncl;
  }
  row_arrive(rs + kRowArrive2);
  merge();  // this CTA's share of the outputs, while the row's other CTAs arrive
  if (!row_wait(rs + kRowArrive2, (uint32_t)S, p.stall_test == 2)) ok = false;
  // Every CTA of the row has its copy of the u histogram by now (each copied it before
  // arriving): clear this CTA's share for the next call.
  uint32_t* gu = p.uhist + (size_t)bq * kHistBins;
  for (int e = split * nt + tid; e < kUBins; e += S * nt) gu[e] = 0u;

  // ---- 3. the row's fine histogram gives B, the bin of the k_sel-th largest t: keys of
  // bins >= B + mb are in, keys of bins [B - mb, B + mb) form the band.  (The scratch
  // holds a copy of the histogram, then the band keys being re-scored and the per-warp K
  // rows, later the band list being ranked.)
  uint32_t* fhs = reinterpret_cast<uint32_t*>(scratch);
  uint8_t* bscr = scratch + kUHistBytes;
  double* bval = reinterpret_cast<double*>(bscr);
  int* bl = reinterpret_cast<int*>(bscr + kBandSmem * 8);
  float* kf = reinterpret_cast<float*>(bscr + kBandSmem * 12);
  async_bins(fhs, gfh);
  sm100::cp_async_wait_all();
  __syncthreads();
  const BinScan bs = scan_bins(fhs, p.k_sel, mb);
  const int B = bs.bin;
  const int n_band = (int)bs.near;
  const int need2 = p.k_sel - (int)bs.above;  // taken from the band: 1 <= need2 <= n_band
  const bool rank_band = need2 < n_band;
  // When every band key is taken the band counts as in.
  const int in_bin = rank_band ? B + mb : B - mb;
  auto in_band = [&](int bb) { return bb >= B - mb && bb < B + mb; };
  uint32_t cin = 0, cband = 0;
#pragma unroll 1
  for (int e = tid; e < own_n; e += nt) {
    const int bb = fb.bin(ot[e]);
    cin += bb >= in_bin;
    cband += rank_band && in_band(bb);
  }
  block_sum2(cin, cband);
  if (tid == 0) rowcnt[split] = cin;  // read by the higher chunks after the third barrier
  // The float64 keys of this chunk's band keys go to the row's band list: up to kBandSmem
  // at a time are listed on chip and taken by the warps in turn (one key per warp).
  if (cband) {
    uint32_t base = 0;
    if (tid == 0) base = atomicAdd(rs + kRowNBand, cband);  // in flight while re-scoring
#pragma unroll 1
    for (uint32_t r0 = 0; r0 < cband; r0 += kBandSmem) {
      const uint32_t rn = min(cband - r0, (uint32_t)kBandSmem);
      block_compact(
          own_n, [&](int e) { return in_band(fb.bin(ot[e])); },
          [&](int at, int e) {
            if ((uint32_t)at - r0 < rn) bl[at - r0] = e;
          });
#pragma unroll 1
      for (int i = warp; i < (int)rn; i += nwarps) {
        const int j = oj[bl[i]];
        const double v = rescore_f64<H, FP8>(p.kv, p.sm_scale, (size_t)b * p.kv.max_len + j,
                                             qv.base, qv.hstride, qv.cstride, rl.dl,
                                             kf + warp * kHeadDim, lane);
        if (lane == 0) {
          bval[i] = v;
          bl[i] = j;
        }
      }
      if (tid == 0) red_s[0][0] = base;
      __syncthreads();
      const uint32_t at0 = red_s[0][0] + r0;
#pragma unroll 1
      for (int i = tid; i < (int)rn; i += nt) {
        const uint32_t slot = at0 + (uint32_t)i;
        if (slot < (uint32_t)p.kv.max_len) {
          p.band_t[rowoff + slot] = bval[i];
          p.band_j[rowoff + slot] = bl[i];
        }
      }
      __syncthreads();
    }
  }
  row_arrive(rs + kRowArrive3);
  if (!row_wait(rs + kRowArrive3, (uint32_t)S, p.stall_test == 2)) ok = false;
  // Every CTA has read the fine histogram: clear this CTA's share for the next call.
  for (int e = split * nt + tid; e < kUBins; e += S * nt) gfh[e] = 0u;

  // ---- 4. the slot of this chunk's first selected position: the selections of the lower
  // chunks (their counts, and the band keys below k0 that the ranking takes)
  uint32_t below = 0, unused = 0;
  // (each count is only added once the band list's loads are also on their way)
  uint32_t lower_cnt[(kSmCountBound + 127) / 128];
#pragma unroll
  for (int u = 0; u < (kSmCountBound + 127) / 128; ++u) {
    const int s2 = tid + u * 128;
    lower_cnt[u] = s2 < split && tid < 128 ? __ldcg(rowcnt + s2) : 0u;
  }
  if (rank_band) {
    // Every CTA ranks the whole band by (key desc, position asc): the top need2 are in.
    // Those of this chunk are marked (~j) in its list.
    const double* gbt = p.band_t + rowoff;
    const int32_t* gbj = p.band_j + rowoff;
    auto take = [&](int je) {
      if (je < k0) ++below;
      else if (je < c_hi) {
        const int e = find_position(oj, own_n, je);
        if (e < own_n) oj[e] = ~je;
      }
    };
    const int nb = min(n_band, (int)p.kv.max_len);
    if (nb <= kBandSmem) {
      unsigned long long* bkey = reinterpret_cast<unsigned long long*>(bval);
      int* bpos = bl;
      for (int e = tid; e < nb; e += nt) {
        bkey[e] = ordered_key64(__ldcg(gbt + e));
        bpos[e] = __ldcg(gbj + e);
      }
      __syncthreads();
      // One warp per band key: its rank is the number of keys ahead of it (key desc,
      // position asc), counted 32 at a time with a ballot.
#pragma unroll 1
      for (int e = warp; e < nb; e += nwarps) {
        const unsigned long long ke = bkey[e];
        const int je = bpos[e];
        int rank = 0;
#pragma unroll 1
        for (int f0 = 0; f0 < nb; f0 += 32) {
          const int f = f0 + lane;
          bool ahead = false;
          if (f < nb) {
            const unsigned long long kf2 = bkey[f];
            ahead = (kf2 > ke) || (kf2 == ke && bpos[f] < je);
          }
          rank += __popc(__ballot_sync(0xffffffffu, ahead));
        }
        if (lane == 0 && rank < need2) take(je);
      }
    } else {
      // A large band (many equal keys): the boundary by radix select over the list.
      __shared__ uint32_t gt_s;
      const unsigned long long vb = block_kth_largest<unsigned long long, 64>(
          nb, need2, [&](int e) { return ordered_key64(__ldcg(gbt + e)); },
          [](int) { return true; }, &gt_s);
      const int take_eq = need2 - (int)gt_s;
      const uint32_t jb_inv = block_kth_largest<uint32_t, 32>(
          nb, take_eq, [&](int e) { return ~(uint32_t)__ldcg(gbj + e); },
          [&](int e) { return ordered_key64(__ldcg(gbt + e)) == vb; }, &gt_s);
      const int jb = (int)~jb_inv;
      for (int e = tid; e < nb; e += nt) {
        const unsigned long long k = ordered_key64(__ldcg(gbt + e));
        const int je = __ldcg(gbj + e);
        if (k > vb || (k == vb && je <= jb)) take(je);
      }
    }
  }
#pragma unroll
  for (int u = 0; u < (kSmCountBound + 127) / 128; ++u) below += lower_cnt[u];
  block_sum2(below, unused);  // also orders the marks before the compaction reads them
  // This chunk's selected positions, in order, from slot `below`.
  block_compact(
      own_n,
      [&](int e) { return oj[e] < 0 || fb.bin(ot[e]) >= in_bin; },
      [&](int at, int e) {
        const uint32_t slot = below + (uint32_t)at;
        const int v = oj[e];
        if (slot < (uint32_t)p.k_sel) out_row[slot] = v < 0 ? ~v : v;
      });
  // The window and the padding after the k_sel selected positions.
  if (split == 0)
    for (int e = p.k_sel + tid; e < width; e += nt) {
      const int v = n_c + (e - p.k_sel);
      out_row[e] = v <= pos ? v : -1;
    }
  return ok;
}

// The whole tail (fuse 1 or 2), called by every thread of every CTA after the stream,
// with the CTA's partial written, its m per head in `own_m` (shared memory; null for a
// CTA that took no tile) and (fuse 2) its u histogram in `uhist_s`.  NW: warps of
// the CTA.  The K/V stages (`stage`, `stage_bytes`) are idle; the first kTailTiles tiles
// of `tile_bytes` take gathered K rows.  Returns false if a wait gave up.
template <int H, bool FP8, int NW, typename Recompute>
__device__ __forceinline__ bool fused_tail(const FullParams& p, uint8_t* stage, uint32_t stage_bytes,
                                           uint32_t tile_bytes, const uint32_t* uhist_s,
                                           const float* own_m, int bq, int b, int split, int pos,
                                           int k0, int k1, const QView& qv, Recompute&& recompute) {
  __shared__ RowLse<H> rl;
  const int S = p.splits1;
  const int n_c = pos - p.window + 1;
  const bool sel_row = p.fuse == 2 && n_c > p.k_sel;
  const int width = p.window + p.k_sel;
  uint32_t* rs = p.rowsync + (size_t)bq * 8;
  uint32_t* gu = p.uhist + (size_t)bq * kHistBins;
  const int c_hi = min(k1, n_c);
  const int chunk_len = sel_row && c_hi > k0 ? c_hi - k0 : 0;
  // The stages hold: the gathered tiles (later the tail's scratch), the row's u
  // histogram, the merge's inputs (when they fit beside a one-piece chunk), then this
  // chunk's bounds (a piece at a time), its candidate positions and their keys.
  const uint32_t tiles = kTailTiles * tile_bytes;
  uint32_t* uh = reinterpret_cast<uint32_t*>(stage + tiles);
  const uint32_t moff = tiles + kUHistBytes;
  const uint32_t fixed = moff + kTailTiles * 128u * 4u;
  uint32_t mbytes = merge_prefetch_bytes<H>(split, S);
  if (fixed + mbytes + 8u * (uint32_t)((chunk_len + 3) & ~3) > stage_bytes) mbytes = 0;
  float* mo = mbytes ? reinterpret_cast<float*>(stage + moff) : nullptr;
  const uint32_t uoff = moff + mbytes;
  const int piece = (int)(((stage_bytes - fixed - mbytes) / 8u) & ~3u);
  float* us = reinterpret_cast<float*>(stage + uoff);
  int* cl = reinterpret_cast<int*>(stage + uoff + 4u * (uint32_t)piece);
  float* t2s = reinterpret_cast<float*>(stage + uoff + 8u * (uint32_t)piece);
  uint32_t* rowmax = p.rowmax + (size_t)bq * kMaxHeads;
  static_assert(NW * 32 * 8 <= kTailTiles * 16384, "the tail's scratch fits the tiles' space");
  bool ok = true;
  __syncthreads();
  if (threadIdx.x < H && own_m) {
    // This CTA's m per head (the value of its partial, still on chip) joins the row's
    // maxima, the reference of the row's lse.
    const float m = own_m[threadIdx.x];
    if (m > -INFINITY) atomicMax(rowmax + threadIdx.x, max_key(m));
  }
  if (sel_row) {
    // This CTA's u histogram added to the row's in one bulk reduction (its writes done
    // and ordered before the barrier's release).
    sm100::fence_proxy_async_smem();
    __syncthreads();
    if (threadIdx.x == 0) {
      sm100::bulk_reduce_add_u32(gu, uhist_s, kUHistBytes);
      sm100::bulk_commit();
      sm100::bulk_wait_all();
      sm100::fence_proxy_async_global();
    }
  }
  row_arrive(rs + kRowArrive1);
  if (!row_wait(rs + kRowArrive1, (uint32_t)S, p.stall_test == 2)) ok = false;
  if (sel_row) {
    // In flight with the partials' loads of row_lse: the row's u histogram and this
    // chunk's first bounds (whichever CTA streamed those keys).
    async_bins(uh, gu);
    async_words(us, p.ubuf + (size_t)bq * p.ld_u + k0, min(piece, chunk_len));
  }
  if (mo) prefetch_merge<H>(p, bq, split, S, mo);  // read at the very end
  row_lse<H>(p.part_ml + (size_t)bq * S * H * 2, rowmax, S, rl, reinterpret_cast<float2*>(stage));
  if (p.fuse == 2 && !sel_row && split == 0)
    write_all_positions(p.sel_idx + (size_t)bq * width, width, pos);
  // The merge needs only the lse and the partials: with a selection it runs while the
  // CTA waits at the row's second barrier, else at the end.
  bool merged = false;
  auto merge = [&]() {
    row_merge<H>(p, bq, split, S, rl, reinterpret_cast<float*>(stage), mo);
    merged = true;
  };
  if (sel_row) {
    sm100::cp_async_wait_all();  // (the merge's partials too)
    __syncthreads();
    const int bk = scan_bins(uh, p.k_sel, 0).bin;
    if (!row_select<H, FP8>(p, stage, us, cl, t2s, piece, bq, b, split, S, k0, c_hi, n_c, pos,
                            bk, rl, qv, recompute, merge))
      ok = false;
  }
  // The index set is complete and visible: the next kernel (a sparse layer, which reads
  // it before waiting for this grid to end) may start while this CTA merges its share.
  sm100::fence_acq_rel_gpu();
  __syncthreads();
  griddep_launch_dependents();
  if (!merged) {
    if (mo) {
      sm100::cp_async_wait_all();
      __syncthreads();
    }
    merge();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // The last CTA of the row to get here leaves the row's counters at zero.
    __threadfence();
    if (atomicAdd(rs + kRowDone, 1u) == (uint32_t)S - 1u) {
      rs[kRowArrive1] = 0u;
      rs[kRowArrive2] = 0u;
      rs[kRowArrive3] = 0u;
      rs[kRowNBand] = 0u;
      rs[kRowDone] = 0u;
      rs[kRowTileSlot] = 0u;
#pragma unroll 1
      for (int hh = 0; hh < H; ++hh) rowmax[hh] = 0u;
      __threadfence();
    }
  }
  return ok;
}

}  // namespace hs2
