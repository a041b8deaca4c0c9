// Selection helpers shared by the selection kernels and the full layer's fused
// selection tail: warp-aggregated slots, a block-wide radix select, and the float64
// re-scoring of one position.
#pragma once

#include "hs2_internal.cuh"

namespace hs2 {

// ----------------------------------------------------------------------------
// float64 selection key of one position, by one warp: max_h(sm_scale * q_h . k_j -
// delta_h) from the stored inputs (K row widened exactly to float32 in the warp's
// shared row kf, the FP8 scale applied to the dot product; each lane takes heads lane,
// lane + 32, ...;
// for H < 32 the lanes split each head's dot product into 32 / H parts, lane = part *
// H + head; four partial sums per lane).  q: the query's bf16 elements, the 8-element
// chunk c of head h at byte q + h * q_hstride + c * q_cstride (shared or global memory,
// 16-byte aligned); dlt: the float64 shifts; kf: the warp's 128 floats of shared memory.
// Every lane returns the key.  krow: the key's K row (bf16, or E4M3 codes with their scale
// ksc), in global or shared memory.
// ----------------------------------------------------------------------------
constexpr int kQLd = kHeadDim + 8;  // padded q row (bf16) in shared memory

// Error-free accumulation of a float32 term p into the pair (s, e) (two-sum): s + e gains
// p exactly, up to the rounding of e itself (a term 2^-24 smaller).
__device__ __forceinline__ void two_sum_acc(float& s, float& e, float p) {
  const float t = s + p;
  const float bp = t - s;
  e += (s - (t - bp)) + (p - bp);
  s = t;
}

template <int H, bool FP8>
__device__ __forceinline__ double rescore_row_f64(const uint8_t* krow, double ksc, float sm_scale,
                                                  const uint8_t* q, int q_hstride, int q_cstride,
                                                  const double* dlt, float* kf, int lane) {
  // Each product q_c k_c is exact in float32 (bf16 x bf16, or bf16 x an E4M3 code: at most
  // 16 significant bits), and the products are summed error-free (two-sum), so the dot
  // product carries about 45 bits before it meets float64; the FP8 scale multiplies the
  // sum in float64.
  constexpr int kParts = H < 32 ? 32 / H : 1;
  constexpr int kSpan = kHeadDim / kParts;
  const int part = kParts > 1 ? lane / H : 0;
  if (FP8) {
    const uint32_t w4 = reinterpret_cast<const uint32_t*>(krow)[lane];
#pragma unroll
    for (int u = 0; u < 4; ++u) kf[4 * lane + u] = e4m3_to_f32((w4 >> (8 * u)) & 0xffu);
  } else {
    const uint2 w4 = reinterpret_cast<const uint2*>(krow)[lane];
    kf[4 * lane] = bf16_bits_to_f32(w4.x & 0xffffu);
    kf[4 * lane + 1] = bf16_bits_to_f32(w4.x >> 16);
    kf[4 * lane + 2] = bf16_bits_to_f32(w4.y & 0xffffu);
    kf[4 * lane + 3] = bf16_bits_to_f32(w4.y >> 16);
  }
  __syncwarp();
  const double scale = (double)sm_scale * ksc;
  double best = -INFINITY;
  for (int h0 = 0; h0 < H; h0 += 32 / kParts) {
    const int h = h0 + (kParts > 1 ? lane % H : lane);
    float s4[4] = {0.f, 0.f, 0.f, 0.f}, e4[4] = {0.f, 0.f, 0.f, 0.f};
    if (h < H) {
      const uint8_t* qh = q + (size_t)h * q_hstride;
#pragma unroll 4
      for (int c = part * kSpan; c < (part + 1) * kSpan; c += 8) {
        const uint4 qv = *reinterpret_cast<const uint4*>(qh + (size_t)(c / 8) * q_cstride);
        const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          two_sum_acc(s4[u], e4[u], bf16_bits_to_f32(qw[u] & 0xffffu) * kf[c + 2 * u]);
          two_sum_acc(s4[u], e4[u], bf16_bits_to_f32(qw[u] >> 16) * kf[c + 2 * u + 1]);
        }
      }
    }
    double d = (((double)s4[0] + (double)s4[1]) + ((double)s4[2] + (double)s4[3])) +
               (((double)e4[0] + (double)e4[1]) + ((double)e4[2] + (double)e4[3]));
#pragma unroll
    for (int o = 16; o >= 32 / kParts && kParts > 1; o >>= 1)
      d += __shfl_xor_sync(0xffffffffu, d, o);
    if (h < H) best = fmax(best, scale * d - dlt[h]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) best = fmax(best, __shfl_xor_sync(0xffffffffu, best, o));
  __syncwarp();  // the warp's next position reuses kf
  return best;
}

// The same for row `row` of the cache.
template <int H, bool FP8>
__device__ __forceinline__ double rescore_f64(const KvView& kv, float sm_scale, size_t row,
                                              const uint8_t* q, int q_hstride, int q_cstride,
                                              const double* dlt, float* kd, int lane) {
  const uint8_t* krow = static_cast<const uint8_t*>(kv.k) + row * (FP8 ? kHeadDim : 2 * kHeadDim);
  const double ksc = FP8 ? (double)__ldg(kv.k_scale + row) : 1.0;
  return rescore_row_f64<H, FP8>(krow, ksc, sm_scale, q, q_hstride, q_cstride, dlt, kd, lane);
}

// Warp-aggregated append to a shared-memory counter: one atomic per warp; returns the
// lane's slot (only meaningful where pred holds).
__device__ __forceinline__ uint32_t warp_slot(bool pred, uint32_t* counter) {
  const unsigned m = __ballot_sync(0xffffffffu, pred);
  const int lane = threadIdx.x & 31;
  uint32_t base = 0;
  if (m) {
    const int leader = __ffs(m) - 1;
    if (lane == leader) base = atomicAdd(counter, (uint32_t)__popc(m));
    base = __shfl_sync(0xffffffffu, base, leader);
  }
  return base + __popc(m & ((1u << lane) - 1u));
}

// Radix select over the elements e in [0, n) with pred(e): the r-th largest
// (1-based) of key(e), a KeyT of KBITS bits, 8 bits per pass.  Returns the key;
// *n_gt receives how many selected elements are strictly greater.  Each pass builds a
// 256-bin shared histogram of the current digit, then warp 0 finds the digit holding
// the r-th element with a warp-wide prefix sum (lane l owns digits 255-8l .. 248-8l).
// Keys known to lie in [lo, hi] share the bits above the highest bit where lo and hi
// differ: those digits are skipped (pass lo = 0, hi = all ones when nothing is known).
template <typename KeyT, int KBITS, typename KeyFn, typename PredFn>
__device__ KeyT block_kth_largest(int n, int r, KeyFn key, PredFn pred, uint32_t* n_gt,
                                  KeyT lo = KeyT(0), KeyT hi = ~KeyT(0)) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t sh_digit, sh_rem, sh_gt;
  const KeyT diff = lo ^ hi;
  if (diff == 0) {  // every key equals lo
    if (threadIdx.x == 0) *n_gt = 0u;
    __syncthreads();
    return lo;
  }
  int top = KBITS - 1;
  while (!((diff >> top) & 1)) --top;
  const int start = (top / 8) * 8;  // lowest bit of the highest digit that varies
  KeyT mask = start + 8 >= KBITS ? KeyT(0) : ~((KeyT(1) << (start + 8)) - 1);
  KeyT prefix = lo & mask;
  uint32_t rem = (uint32_t)r, gt = 0;
  for (int shift = start; shift >= 0; shift -= 8) {
    for (int e = threadIdx.x; e < 256; e += blockDim.x) hist[e] = 0u;
    if (threadIdx.x == 0) {
      sh_digit = 0u;
      sh_rem = rem;
      sh_gt = 0u;
    }
    __syncthreads();
    // Keys of one pass share most of their digits (the candidates come from one bin),
    // so lanes with the same digit are combined first: one shared atomic per distinct
    // digit per warp instead of one per key on the same address.
    const int n_r = (n + 31) & ~31;  // whole warps take part in the match
    for (int e = threadIdx.x; e < n_r; e += blockDim.x) {
      bool take = false;
      uint32_t digit = 0;
      if (e < n && pred(e)) {
        const KeyT k = key(e);
        take = (k & mask) == prefix;
        digit = (uint32_t)(k >> shift) & 255u;
      }
      const uint32_t tag = take ? digit : 256u;
      const unsigned same = __match_any_sync(0xffffffffu, tag);
      if (take && (threadIdx.x & 31) == __ffs(same) - 1) atomicAdd(&hist[digit], __popc(same));
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      uint32_t c[8], s = 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        c[u] = hist[255 - 8 * lane - u];
        s += c[u];
      }
      uint32_t incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const uint32_t excl = incl - s;
      if (excl < rem && rem <= incl) {
        uint32_t cum = excl;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (cum + c[u] >= rem) {
            sh_digit = (uint32_t)(255 - 8 * lane - u);
            sh_rem = rem - cum;
            sh_gt = cum;
            break;
          }
          cum += c[u];
        }
      }
    }
    __syncthreads();
    prefix |= (KeyT)sh_digit << shift;
    mask |= (KeyT)255 << shift;
    rem = sh_rem;
    gt += sh_gt;
    __syncthreads();
  }
  if (threadIdx.x == 0) *n_gt = gt;
  __syncthreads();
  return prefix;
}

}  // namespace hs2
