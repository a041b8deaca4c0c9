// Appending new tokens to the cache: the step before the full layer in a decode loop
// (the pages' KV cache, possibly FP8: "Luo Fuli Teases Xiaomi MiMo-V3 Architecture ...",
// paragraph on cost at one million tokens).  One CTA per sequence: each warp takes whole
// rows (K or V of one new token, 128 values, four per lane); an FP8 cache stores the
// row's E4M3 codes and its per-token scale s = amax / 448 (code = x / s rounded to
// nearest even with saturation, both divisions IEEE float32; an all-zero row gets
// s = 1).  The CTA reads the sequence's length once and grows it after every row is
// written, so no other CTA reads or writes that length.  The next kernel may start only
// once every CTA has written its rows and length.
#include <cuda_fp8.h>

#include "hs2_internal.cuh"

namespace hs2 {

constexpr int kAppendThreads = 256;

__global__ void __launch_bounds__(kAppendThreads) kv_append_kernel(AppendParams p) {
  griddep_wait();  // earlier kernels may still read the lengths and the cache
  const int b = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int L = p.lens[b];
  const bool fits = L >= 0 && L + p.n_new <= p.max_len;
  if (!fits) {
    if (threadIdx.x == 0) set_status(p.status, HS2_ERR_BAD_LENGTH);
    return;  // (an exiting CTA counts as having let the next kernel start)
  }
  const int rows = 2 * p.n_new;  // K then V of each new token
  for (int r = warp; r < rows; r += kAppendThreads / 32) {
    const int i = r >> 1;
    const bool is_v = r & 1;
    const uint16_t* src = (is_v ? p.v_new : p.k_new) + ((size_t)b * p.n_new + i) * kHeadDim;
    const size_t row = (size_t)b * p.max_len + L + i;
    const uint2 w = *reinterpret_cast<const uint2*>(src + 4 * lane);  // 4 bf16 per lane
    if (!p.fp8) {
      uint16_t* dst = static_cast<uint16_t*>(is_v ? p.v : p.k) + row * kHeadDim;
      *reinterpret_cast<uint2*>(dst + 4 * lane) = w;
      continue;
    }
    const float x[4] = {bf16_bits_to_f32(w.x & 0xffffu), bf16_bits_to_f32(w.x >> 16),
                        bf16_bits_to_f32(w.y & 0xffffu), bf16_bits_to_f32(w.y >> 16)};
    float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
    amax = warp_max(amax);
    const float s = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
    const float2 y01 = make_float2(__fdiv_rn(x[0], s), __fdiv_rn(x[1], s));
    const float2 y23 = make_float2(__fdiv_rn(x[2], s), __fdiv_rn(x[3], s));
    const uint32_t c01 = __nv_cvt_float2_to_fp8x2(y01, __NV_SATFINITE, __NV_E4M3);
    const uint32_t c23 = __nv_cvt_float2_to_fp8x2(y23, __NV_SATFINITE, __NV_E4M3);
    uint8_t* dst = static_cast<uint8_t*>(is_v ? p.v : p.k) + row * kHeadDim;
    *reinterpret_cast<uint32_t*>(dst + 4 * lane) = (c01 & 0xffffu) | (c23 << 16);
    if (lane == 0) (is_v ? p.v_scale : p.k_scale)[row] = s;
  }
  __syncthreads();
  if (threadIdx.x == 0) p.lens[b] = L + p.n_new;
  // The next kernel may read the lengths and the cache before it waits for this one (the
  // tensor-core sparse layer does): only the complete, visible rows and lengths let it start.
  __threadfence();
  __syncthreads();
  griddep_launch_dependents();
}

cudaError_t launch_kv_append(const AppendParams& p, int batch, cudaStream_t st) {
  return launch_pdl(kv_append_kernel, dim3(batch), dim3(kAppendThreads), 0, st, p);
}

}  // namespace hs2
