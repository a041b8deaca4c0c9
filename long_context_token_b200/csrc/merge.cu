// Merge of split partials (m, l, unnormalised o) into the normalised output and the
// per-head log-sum-exp, for the full layer and the sparse layers.
//
//   out_h = sum_s w_sh o_sh,  w_sh = e^(m_sh - M_h) / L_h,  L_h = sum_s l_sh e^(m_sh - M_h),
//   lse_h = M_h + ln L_h
// (base 2 instead of e when the partials were produced in the log2 domain).
//
// Grid (bq, h): one CTA per (sequence/token, head), 128 x G threads (G = ceil(S / 8),
// at most 8).  Thread (g, d) first requests dimension d of the partials s = g, g + G,
// ... (eight at once); meanwhile warp 0 loads the (m, l) pairs, reduces M and L over
// the splits (float64 sum) and stages the weights in shared memory.  Each thread then
// sums its partials and the G partial sums are added in shared memory.
#include "hs2_internal.cuh"

namespace hs2 {

constexpr int kMergeMaxGroups = 8;

template <bool LOG2>
__global__ void __launch_bounds__(kHeadDim * kMergeMaxGroups) merge_splits_kernel(MergeParams p) {
  extern __shared__ float w[];  // [splits] weights, [G][128] partial sums, [splits][2] (m, l)
  const int bq = blockIdx.x, h = blockIdx.y;
  const int H = p.h, S = p.splits;
  const int G = blockDim.x / kHeadDim;
  float* acc_s = w + ((S + 3) & ~3);
  float* ml_s = acc_s + G * kHeadDim;
  const float* pml = p.part_ml + (size_t)bq * S * H * 2;
  const float* po = p.part_o + (size_t)bq * S * H * kHeadDim;
  griddep_wait();
  // The importance pass that may follow takes nothing from this kernel until it exits,
  // so it may start now.
  griddep_launch_dependents();
  // The first eight partials of this thread's dimension are requested before the
  // weights are known, so the (m, l) and o loads share one memory round trip.
  const int d = threadIdx.x % kHeadDim, g = threadIdx.x / kHeadDim;
  const float* src = po + (size_t)h * kHeadDim + d;
  const size_t stride = (size_t)H * kHeadDim;
  float v0[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) v0[u] = g + u * G < S ? __ldcg(src + (size_t)(g + u * G) * stride) : 0.f;
  if (threadIdx.x < 32) {
    // One pass over the (m, l) pairs (a single memory round trip), kept in shared memory.
    const int lane = threadIdx.x;
    float M = -INFINITY;
#pragma unroll 4
    for (int s = lane; s < S; s += 32) {
      const float2 v = __ldcg(reinterpret_cast<const float2*>(pml + ((size_t)s * H + h) * 2));
      ml_s[2 * s] = v.x;
      ml_s[2 * s + 1] = v.y;
      if (v.y > 0.f) M = fmaxf(M, v.x);
    }
    M = warp_max(M);
    double Ls = 0.0;
    if (M != -INFINITY) {
      for (int s = lane; s < S; s += 32) {
        const float m = ml_s[2 * s], l = ml_s[2 * s + 1];
        if (l > 0.f) Ls += (double)l * (LOG2 ? exp2((double)m - M) : exp((double)m - M));
      }
    }
    Ls = warp_sum_d(Ls);
    const float il = Ls > 0.0 ? (float)(1.0 / Ls) : 0.f;
    for (int s = lane; s < S; s += 32) {
      float wt = 0.f;
      const float m = ml_s[2 * s], l = ml_s[2 * s + 1];
      if (M != -INFINITY && l > 0.f) wt = (LOG2 ? exp2f(m - M) : expf(m - M)) * il;
      w[s] = wt;
    }
    if (lane == 0) {
      double lse = -INFINITY;
      if (Ls > 0.0) lse = LOG2 ? ((double)M + log2(Ls)) * 0.69314718055994530942 : M + log(Ls);
      if (p.lse64) p.lse64[(size_t)bq * H + h] = lse;
      if (p.lse_out) p.lse_out[(size_t)bq * H + h] = (float)lse;
    }
  }
  __syncthreads();
  float acc = 0.f;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int s = g + u * G;
    if (s < S) {
      const float wt = w[s];
      if (wt != 0.f) acc = fmaf(wt, v0[u], acc);
    }
  }
  int s = g + 8 * G;
  for (; s + 7 * G < S; s += 8 * G) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = __ldcg(src + (size_t)(s + u * G) * stride);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float wt = w[s + u * G];
      if (wt != 0.f) acc = fmaf(wt, v[u], acc);
    }
  }
  for (; s < S; s += G) {
    const float wt = w[s];
    if (wt != 0.f) acc = fmaf(wt, __ldcg(src + (size_t)s * stride), acc);
  }
  acc_s[g * kHeadDim + d] = acc;
  __syncthreads();
  if (g == 0) {
    float t = 0.f;
    for (int k = 0; k < G; ++k) t += acc_s[k * kHeadDim + d];
    p.out[((size_t)bq * H + h) * kHeadDim + d] = t;
  }
}

cudaError_t launch_merge(const MergeParams& p, int bq, bool log2_domain, cudaStream_t st) {
  int G = (p.splits + 7) / 8;
  if (G > kMergeMaxGroups) G = kMergeMaxGroups;
  if (G < 1) G = 1;
  const size_t smem =
      (((size_t)p.splits + 3) / 4 * 4 + (size_t)G * kHeadDim + 2 * (size_t)p.splits) * sizeof(float);
  if (smem > 200 * 1024) return cudaErrorInvalidValue;
  static size_t attr_set[2] = {0, 0};
  const int which = log2_domain ? 1 : 0;
  if (smem > 48 * 1024 && smem > attr_set[which]) {
    cudaError_t e = log2_domain
        ? cudaFuncSetAttribute(merge_splits_kernel<true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)
        : cudaFuncSetAttribute(merge_splits_kernel<false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_set[which] = smem;
  }
  dim3 grid(bq, p.h);
  return log2_domain
             ? launch_pdl(merge_splits_kernel<true>, grid, dim3(kHeadDim * G), smem, st, p)
             : launch_pdl(merge_splits_kernel<false>, grid, dim3(kHeadDim * G), smem, st, p);
}

}  // namespace hs2
