// Reusing sparse-attention layer of the hybrid block: the layer's own queries attend
// only to the positions of the shared index set, read from the shared KV cache
// (web coverage of HySparse2: toolnavs article 2080, fr "Ce que fait HySparse2",
// KV Reuse paragraph -- the sparse layers reuse the full layer's KV cache and its
// selected indices).  Softmax over the selected rows only; -1 slots are skipped.
//
// Grid: (splits4, batch * n_q).  CTA (split, bq) gathers index entries
// [split * chunk4, (split + 1) * chunk4) of its row with 16-byte row loads; the last
// CTA of each row merges the splits (ticket counter, no spin-wait).
#include "tile_simt.cuh"

namespace hs2 {

template <int H, bool FP8>
__global__ void __launch_bounds__(kThreads) sparse_attn_simt_kernel(SparseParams p) {
  extern __shared__ __align__(16) float smem[];
  SimtSmem s = carve_simt(smem, H);
  const int split = blockIdx.x, bq = blockIdx.y;
  const int b = bq / p.n_q;
  const int L = seq_len(p.kv, b, p.n_q, p.status, false);
  const int e0 = split * p.chunk4;
  const int e1 = min(e0 + p.chunk4, p.idx_width);
  const int32_t* idx = p.idx + (size_t)bq * p.idx_width;

  load_q_scaled<H>(s.qs, p.q + (size_t)bq * H * kHeadDim, p.sm_scale);
  for (int hd = threadIdx.x; hd < H; hd += kThreads) {
    s.m_run[hd] = -INFINITY;
    s.l_run[hd] = 0.f;
  }
  float acc[H / 2];
#pragma unroll
  for (int r = 0; r < H / 2; ++r) acc[r] = 0.f;
  const size_t row_base = (size_t)b * p.kv.max_len;
  for (int t0 = e0; t0 < e1; t0 += kTile) {
    __syncthreads();
    if (threadIdx.x < kTile) {
      const int e = t0 + threadIdx.x;
      int row = -1;
      if (e < e1) {
        const int j = __ldg(idx + e);
        if (j >= 0 && j < L) row = (int)(row_base + j);
        else if (j != -1) set_status(p.status, HS2_ERR_INDEX_OUT_OF_RANGE);
      }
      s.rowidx[threadIdx.x] = row;
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
  const size_t pidx = (size_t)bq * p.splits4 + split;
  write_partial<H>(s, acc, p.part_o + pidx * H * kHeadDim, p.part_ml + pidx * H * 2);
  if (!arrive_last(p.tickets + bq, p.splits4)) return;
  double* lse_d = reinterpret_cast<double*>(s.ks);
  merge_partials<H>(p.part_o + (size_t)bq * p.splits4 * H * kHeadDim,
                    p.part_ml + (size_t)bq * p.splits4 * H * 2, p.splits4,
                    p.out + (size_t)bq * H * kHeadDim, lse_d, s.vs);
}

template <int H, bool FP8>
static cudaError_t launch_sparse_t(const SparseParams& p, int batch, cudaStream_t st) {
  const size_t smem = simt_smem_bytes(H);
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(sparse_attn_simt_kernel<H, FP8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  sparse_attn_simt_kernel<H, FP8><<<dim3(p.splits4, batch * p.n_q), kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

template <bool FP8>
static cudaError_t launch_sparse_h(const SparseParams& p, int batch, cudaStream_t st) {
  switch (p.h) {
    case 16: return launch_sparse_t<16, FP8>(p, batch, st);
    case 32: return launch_sparse_t<32, FP8>(p, batch, st);
    case 48: return launch_sparse_t<48, FP8>(p, batch, st);
    case 64: return launch_sparse_t<64, FP8>(p, batch, st);
    case 80: return launch_sparse_t<80, FP8>(p, batch, st);
    case 96: return launch_sparse_t<96, FP8>(p, batch, st);
    case 112: return launch_sparse_t<112, FP8>(p, batch, st);
    case 128: return launch_sparse_t<128, FP8>(p, batch, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_sparse_attn(const SparseParams& p, int batch, cudaStream_t st) {
  return p.kv.fp8 ? launch_sparse_h<true>(p, batch, st) : launch_sparse_h<false>(p, batch, st);
}

}  // namespace hs2
