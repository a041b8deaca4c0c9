// CUDA-core building blocks: 32-row K/V tiles staged as float32 in shared memory,
// the QK^T tile, the online-softmax update and the P.V accumulation.  Used by the full layer (contiguous rows), the importance pass and
// the sparse layers (gathered rows).
#pragma once

#include "hs2_internal.cuh"

namespace hs2 {

constexpr int kTile = 32;      // rows per tile
constexpr int kThreads = 256;  // threads per CTA of the SIMT kernels
constexpr int kKsLd = kHeadDim + 1;  // padded row stride of the staged K tile

// Dynamic shared memory of a SIMT attention CTA with H heads.
__host__ __device__ constexpr size_t simt_smem_bytes(int H) {
  return sizeof(float) * ((size_t)H * kHeadDim      // q (pre-scaled)
                          + kTile * kKsLd            // K tile
                          + kTile * kHeadDim         // V tile
                          + (size_t)H * kTile        // S / P tile
                          + 4 * (size_t)H)           // m, l (two floats), alpha
         + sizeof(int) * kTile;                      // row index of each tile row
}

struct SimtSmem {
  float* qs;
  float* ks;
  float* vs;
  float* S;
  float* m_run;
  float* l_run;
  float* l_err;  // trailing float of l (l = l_run + l_err, summed without loss)
  float* alpha;
  int* rowidx;
};

__device__ __forceinline__ SimtSmem carve_simt(float* sm, int H) {
  SimtSmem s;
  s.qs = sm;
  s.ks = s.qs + H * kHeadDim;
  s.vs = s.ks + kTile * kKsLd;
  s.S = s.vs + kTile * kHeadDim;
  s.m_run = s.S + H * kTile;
  s.l_run = s.m_run + H;
  s.l_err = s.l_run + H;
  s.alpha = s.l_err + H;
  s.rowidx = reinterpret_cast<int*>(s.alpha + H);
  return s;
}

// q (bf16 bits) of one (sequence, token) -> shared float, times sm_scale.
template <int H>
__device__ __forceinline__ void load_q_scaled(float* qs, const uint16_t* q, float sm_scale) {
  for (int e = threadIdx.x; e < H * kHeadDim; e += kThreads)
    qs[e] = bf16_bits_to_f32(q[e]) * sm_scale;
}

// Stage kTile cache rows into shared float32 (row r of `dst` has stride ld).
// rowidx[r] is the flat row (b * max_len + j) or -1 for an absent row (zeros).
// FP8 rows are decoded and multiplied by their per-token scale.
template <bool FP8>
__device__ __forceinline__ void load_rows(float* dst, int ld, const void* base,
                                          const float* scale, const int* rowidx) {
  if (!FP8) {
    const uint16_t* src = static_cast<const uint16_t*>(base);
    for (int v = threadIdx.x; v < kTile * 16; v += kThreads) {
      const int r = v >> 4, c = (v & 15) * 8;
      const int row = rowidx[r];
      float* d = dst + r * ld + c;
      if (row >= 0) {
        const uint4 x = __ldg(reinterpret_cast<const uint4*>(src + (size_t)row * kHeadDim + c));
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          d[2 * e] = bf16_bits_to_f32(w[e] & 0xffffu);
          d[2 * e + 1] = bf16_bits_to_f32(w[e] >> 16);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) d[e] = 0.f;
      }
    }
  } else {
    const uint8_t* src = static_cast<const uint8_t*>(base);
    for (int v = threadIdx.x; v < kTile * 8; v += kThreads) {
      const int r = v >> 3, c = (v & 7) * 16;
      const int row = rowidx[r];
      float* d = dst + r * ld + c;
      if (row >= 0) {
        const uint4 x = __ldg(reinterpret_cast<const uint4*>(src + (size_t)row * kHeadDim + c));
        const float sc = __ldg(scale + row);
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
#pragma unroll
          for (int t = 0; t < 4; ++t) d[4 * e + t] = e4m3_to_f32((w[e] >> (8 * t)) & 0xffu) * sc;
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) d[e] = 0.f;
      }
    }
  }
}

// S[h][r] = qs[h] . ks[r] for every head and tile row; -inf for absent rows.
template <int H>
__device__ __forceinline__ void qk_tile(const SimtSmem& s) {
  constexpr int R = H / 8;  // heads per thread
  const int key = threadIdx.x & 31, hg = threadIdx.x >> 5;
  float acc[R];
#pragma unroll
  for (int r = 0; r < R; ++r) acc[r] = 0.f;
  const float* kr = s.ks + key * kKsLd;
#pragma unroll 4
  for (int c = 0; c < kHeadDim; ++c) {
    const float kv = kr[c];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = fmaf(s.qs[(hg + 8 * r) * kHeadDim + c], kv, acc[r]);
  }
  const bool valid = s.rowidx[key] >= 0;
#pragma unroll
  for (int r = 0; r < R; ++r) s.S[(hg + 8 * r) * kTile + key] = valid ? acc[r] : -INFINITY;
}

// Online-softmax update of one tile: S <- exp(S - m), l and alpha updated.  The
// reference m moves only when a logit exceeds it by more than kLazyRescale (or on the
// first key), so l and O are rescaled a handful of times per chunk, and l is summed
// without loss (two-sum): the partial's l carries little more than the rounding of the
// exponentials, which the float64 lse of the selection relies on.
constexpr float kLazyRescale = 8.f;  // p <= e^8 between rescales
template <int H>
__device__ __forceinline__ void softmax_tile(const SimtSmem& s) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  for (int hd = w; hd < H; hd += kThreads / 32) {
    const float x = s.S[hd * kTile + lane];
    const float m_old = s.m_run[hd];
    const float tmax = warp_max(x);
    const float m_new = (m_old == -INFINITY || tmax > m_old + kLazyRescale) ? fmaxf(m_old, tmax)
                                                                           : m_old;
    float pr = 0.f, al = 1.f;
    if (m_new != -INFINITY) {
      pr = expf(x - m_new);
      if (m_new != m_old) al = expf(m_old - m_new);
    }
    const float sum = warp_sum(pr);
    s.S[hd * kTile + lane] = pr;
    __syncwarp();
    if (lane == 0) {
      s.alpha[hd] = al;
      s.m_run[hd] = m_new;
      float l = s.l_run[hd] * al, e = s.l_err[hd] * al;
      const float t = l + sum, bp = t - l;
      e += (l - (t - bp)) + (sum - bp);
      s.l_run[hd] = t;
      s.l_err[hd] = e;
    }
  }
}

// acc[r] (head hg2 + 2r, dimension d) = acc * alpha + sum_r P[h][r] V[r][d].
template <int H>
__device__ __forceinline__ void pv_tile(const SimtSmem& s, float* acc) {
  const int d = threadIdx.x & (kHeadDim - 1), hg2 = threadIdx.x >> 7;
#pragma unroll
  for (int r = 0; r < H / 2; ++r) {
    const int hd = hg2 + 2 * r;
    float a = acc[r] * s.alpha[hd];
    const float* pr = s.S + hd * kTile;
#pragma unroll 8
    for (int j = 0; j < kTile; ++j) a = fmaf(pr[j], s.vs[j * kHeadDim + d], a);
    acc[r] = a;
  }
}

// Selection shift delta_h = lse_h - min_h' lse_h' of one (sequence, token), from the
// full layer's float64 lse (every thread of the block calls this).
__device__ __forceinline__ void load_delta(const double* lse64, int H, float* d32, double* d64) {
  // Warp 0 loads every head's lse at once (one memory round trip) and reduces the min.
  if (threadIdx.x < 32) {
    constexpr int kPerLane = kMaxHeads / 32;
    double v[kPerLane];
    double m = INFINITY;
#pragma unroll
    for (int u = 0; u < kPerLane; ++u) {
      const int h = (int)threadIdx.x + 32 * u;
      v[u] = h < H ? __ldcg(lse64 + h) : INFINITY;
      m = fmin(m, v[u]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmin(m, __shfl_xor_sync(0xffffffffu, m, o));
#pragma unroll
    for (int u = 0; u < kPerLane; ++u) {
      const int h = (int)threadIdx.x + 32 * u;
      if (h < H) {
        const double d = v[u] - m;
        if (d32) d32[h] = (float)d;
        if (d64) d64[h] = d;
      }
    }
  }
  __syncthreads();
}

// Write this split's partial state (m, l, unnormalised o).
template <int H>
__device__ __forceinline__ void write_partial(const SimtSmem& s, const float* acc,
                                              float* part_o, float* part_ml) {
  const int d = threadIdx.x & (kHeadDim - 1), hg2 = threadIdx.x >> 7;
#pragma unroll
  for (int r = 0; r < H / 2; ++r) part_o[(hg2 + 2 * r) * kHeadDim + d] = acc[r];
  for (int hd = threadIdx.x; hd < H; hd += kThreads) {
    part_ml[2 * hd] = s.m_run[hd];
    part_ml[2 * hd + 1] = s.l_run[hd] + s.l_err[hd];
  }
}

}  // namespace hs2
