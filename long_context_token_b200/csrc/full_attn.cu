// Full-attention layer of the hybrid block: split-K flash-decode over every key a
// query token can see, then a merge of the splits into the output and the per-head
// log-sum-exp (web coverage of HySparse2: toolnavs article 2080, fr "Ce que fait
// HySparse2" -- the full layer attends over the whole context and its scores drive
// the selection; MQA per "Les chiffres mesurés").
//
// Grid: (splits1, batch * n_q).  CTA (split, bq) owns keys
// [split * chunk1, (split + 1) * chunk1) of its sequence, clipped to [0, p], and
// writes that chunk's partial (m, l, o); merge.cu combines the chunks.
#include "tile_simt.cuh"

namespace hs2 {

template <int H, bool FP8>
__global__ void __launch_bounds__(kThreads) full_attn_simt_kernel(FullParams p) {
  extern __shared__ __align__(16) float smem[];
  SimtSmem s = carve_simt(smem, H);
  griddep_wait();
  const int split = blockIdx.x, bq = blockIdx.y;
  const int b = bq / p.n_q, i = bq % p.n_q;
  const int L = seq_len(p.kv, b, p.n_q, p.status, split == 0 && i == 0);
  const int pos = L - p.n_q + i;
  const int k0 = split * p.chunk1;
  const int k1 = min(k0 + p.chunk1, pos + 1);

  load_q_scaled<H>(s.qs, p.q + (size_t)bq * H * kHeadDim, p.sm_scale);
  for (int hd = threadIdx.x; hd < H; hd += kThreads) {
    s.m_run[hd] = -INFINITY;
    s.l_run[hd] = 0.f;
    s.l_err[hd] = 0.f;
  }
  float acc[H / 2];
#pragma unroll
  for (int r = 0; r < H / 2; ++r) acc[r] = 0.f;

  const size_t row_base = (size_t)b * p.kv.max_len;
  for (int j0 = k0; j0 < k1; j0 += kTile) {
    __syncthreads();
    if (threadIdx.x < kTile) {
      const int j = j0 + threadIdx.x;
      s.rowidx[threadIdx.x] = j < k1 ? (int)(row_base + j) : -1;
    }
    __syncthreads();
    load_rows<FP8>(s.ks, kKsLd, p.kv.k, p.kv.k_scale, s.rowidx);
    load_rows<FP8>(s.vs, kHeadDim, p.kv.v, p.kv.v_scale, s.rowidx);
    __syncthreads();
    qk_tile<H>(s);
    __syncthreads();
    softmax_tile<H>(s);
    __syncthreads();
    pv_tile<H>(s, acc);
  }
  __syncthreads();
  const size_t pidx = (size_t)bq * p.splits1 + split;
  write_partial<H>(s, acc, p.part_o + pidx * H * kHeadDim, p.part_ml + pidx * H * 2);

}

template <int H, bool FP8>
static cudaError_t launch_full_t(const FullParams& p, int batch, cudaStream_t st) {
  const size_t smem = simt_smem_bytes(H);
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(full_attn_simt_kernel<H, FP8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  dim3 grid(p.splits1, batch * p.n_q);
  return launch_pdl(full_attn_simt_kernel<H, FP8>, grid, dim3(kThreads), smem, st, p);
}

template <bool FP8>
static cudaError_t launch_full_h(const FullParams& p, int batch, cudaStream_t st) {
  switch (p.h) {
    case 16: return launch_full_t<16, FP8>(p, batch, st);
    case 32: return launch_full_t<32, FP8>(p, batch, st);
    case 48: return launch_full_t<48, FP8>(p, batch, st);
    case 64: return launch_full_t<64, FP8>(p, batch, st);
    case 80: return launch_full_t<80, FP8>(p, batch, st);
    case 96: return launch_full_t<96, FP8>(p, batch, st);
    case 112: return launch_full_t<112, FP8>(p, batch, st);
    case 128: return launch_full_t<128, FP8>(p, batch, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_full_attn(const FullParams& p, int batch, cudaStream_t st) {
  return p.kv.fp8 ? launch_full_h<true>(p, batch, st) : launch_full_h<false>(p, batch, st);
}

}  // namespace hs2
