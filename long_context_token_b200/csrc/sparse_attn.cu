// Reusing sparse-attention layer of the hybrid block: the layer's own queries attend
// only to the positions of the shared index set, read from the shared KV cache
// (web coverage of HySparse2: toolnavs article 2080, fr "Ce que fait HySparse2",
// KV Reuse paragraph -- the sparse layers reuse the full layer's KV cache and its
// selected indices).  Softmax over the selected rows only; -1 slots are skipped.
//
// Grid: (ceil(idx_width / 64), batch * n_q).  CTA (split, bq) takes index entries
// [64 split, 64 split + 64) of its row, gathers the 64 K and V rows with 16-byte loads
// (all issued before the first one is used, so the chunk costs one memory round trip),
// and writes the chunk's partial (m, l, o); merge.cu combines the chunks.
#include "hs2_internal.cuh"

namespace hs2 {

constexpr int kSpRows = 64;          // index entries per CTA
constexpr int kSpThreads = 256;
constexpr int kSpKLd = kHeadDim + 1;  // padded K row stride (conflict-free column reads)

__host__ __device__ constexpr size_t sparse_smem_bytes(int H) {
  return sizeof(float) * ((size_t)H * kHeadDim + kSpRows * kSpKLd + kSpRows * kHeadDim +
                          (size_t)H * kSpRows) +
         sizeof(int) * kSpRows;
}

template <int H, bool FP8>
__global__ void __launch_bounds__(kSpThreads) sparse_attn_kernel(SparseParams p) {
  extern __shared__ __align__(16) float smem[];
  float* qs = smem;                          // [H][128], pre-scaled by sm_scale
  float* ks = qs + H * kHeadDim;             // [64][129]
  float* vs = ks + kSpRows * kSpKLd;         // [64][128]
  float* S = vs + kSpRows * kHeadDim;        // [H][64] logits, then probabilities
  int* rowidx = reinterpret_cast<int*>(S + H * kSpRows);
  griddep_wait();
  const int tid = threadIdx.x;
  const int split = blockIdx.x, bq = blockIdx.y;
  const int b = bq / p.n_q;
  const int L = seq_len(p.kv, b, p.n_q, p.status, false);
  const int32_t* idx = p.idx + (size_t)bq * p.idx_width;
  const size_t row_base = (size_t)b * p.kv.max_len;

  if (tid < kSpRows) {
    const int e = split * kSpRows + tid;
    int row = -1;
    if (e < p.idx_width) {
      const int j = __ldg(idx + e);
      if (j >= 0 && j < L) row = (int)(row_base + j);
      else if (j != -1) set_status(p.status, HS2_ERR_INDEX_OUT_OF_RANGE);
    }
    rowidx[tid] = row;
  }
  __syncthreads();

  // Gather: every load of the chunk is issued first, then converted to float32.
  if (!FP8) {
    constexpr int kVec = kSpRows * 16 / kSpThreads;  // 16-byte vectors per thread per tensor
    const uint16_t* kb = static_cast<const uint16_t*>(p.kv.k);
    const uint16_t* vb = static_cast<const uint16_t*>(p.kv.v);
    uint4 kx[kVec], vx[kVec];
#pragma unroll
    for (int u = 0; u < kVec; ++u) {
      const int v = tid + u * kSpThreads, r = v >> 4, c = (v & 15) * 8;
      const int row = rowidx[r];
      kx[u] = row >= 0 ? __ldg(reinterpret_cast<const uint4*>(kb + (size_t)row * kHeadDim + c))
                       : make_uint4(0, 0, 0, 0);
      vx[u] = row >= 0 ? __ldg(reinterpret_cast<const uint4*>(vb + (size_t)row * kHeadDim + c))
                       : make_uint4(0, 0, 0, 0);
    }
    for (int e = tid; e < H * kHeadDim; e += kSpThreads)
      qs[e] = bf16_bits_to_f32(p.q[(size_t)bq * H * kHeadDim + e]) * p.sm_scale;
#pragma unroll
    for (int u = 0; u < kVec; ++u) {
      const int v = tid + u * kSpThreads, r = v >> 4, c = (v & 15) * 8;
      const uint32_t kw[4] = {kx[u].x, kx[u].y, kx[u].z, kx[u].w};
      const uint32_t vw[4] = {vx[u].x, vx[u].y, vx[u].z, vx[u].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        ks[r * kSpKLd + c + 2 * q] = bf16_bits_to_f32(kw[q] & 0xffffu);
        ks[r * kSpKLd + c + 2 * q + 1] = bf16_bits_to_f32(kw[q] >> 16);
        vs[r * kHeadDim + c + 2 * q] = bf16_bits_to_f32(vw[q] & 0xffffu);
        vs[r * kHeadDim + c + 2 * q + 1] = bf16_bits_to_f32(vw[q] >> 16);
      }
    }
  } else {
    constexpr int kVec = kSpRows * 8 / kSpThreads;
    const uint8_t* kb = static_cast<const uint8_t*>(p.kv.k);
    const uint8_t* vb = static_cast<const uint8_t*>(p.kv.v);
    uint4 kx[kVec], vx[kVec];
    float ksc[kVec], vsc[kVec];
#pragma unroll
    for (int u = 0; u < kVec; ++u) {
      const int v = tid + u * kSpThreads, r = v >> 3, c = (v & 7) * 16;
      const int row = rowidx[r];
      kx[u] = row >= 0 ? __ldg(reinterpret_cast<const uint4*>(kb + (size_t)row * kHeadDim + c))
                       : make_uint4(0, 0, 0, 0);
      vx[u] = row >= 0 ? __ldg(reinterpret_cast<const uint4*>(vb + (size_t)row * kHeadDim + c))
                       : make_uint4(0, 0, 0, 0);
      ksc[u] = row >= 0 ? __ldg(p.kv.k_scale + row) : 0.f;
      vsc[u] = row >= 0 ? __ldg(p.kv.v_scale + row) : 0.f;
    }
    for (int e = tid; e < H * kHeadDim; e += kSpThreads)
      qs[e] = bf16_bits_to_f32(p.q[(size_t)bq * H * kHeadDim + e]) * p.sm_scale;
#pragma unroll
    for (int u = 0; u < kVec; ++u) {
      const int v = tid + u * kSpThreads, r = v >> 3, c = (v & 7) * 16;
      const uint32_t kw[4] = {kx[u].x, kx[u].y, kx[u].z, kx[u].w};
      const uint32_t vw[4] = {vx[u].x, vx[u].y, vx[u].z, vx[u].w};
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          ks[r * kSpKLd + c + 4 * q + t] = e4m3_to_f32((kw[q] >> (8 * t)) & 0xffu) * ksc[u];
          vs[r * kHeadDim + c + 4 * q + t] = e4m3_to_f32((vw[q] >> (8 * t)) & 0xffu) * vsc[u];
        }
    }
  }
  __syncthreads();

  // S[h][r] = q_h . k_r: thread (key r = tid % 64, head group tid / 64).
  {
    constexpr int R = H / 4;
    const int key = tid & (kSpRows - 1), hg = tid >> 6;
    float acc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) acc[r] = 0.f;
    const float* kr = ks + key * kSpKLd;
#pragma unroll 4
    for (int c = 0; c < kHeadDim; ++c) {
      const float kv = kr[c];
#pragma unroll
      for (int r = 0; r < R; ++r) acc[r] = fmaf(qs[(hg + 4 * r) * kHeadDim + c], kv, acc[r]);
    }
    const bool valid = rowidx[key] >= 0;
#pragma unroll
    for (int r = 0; r < R; ++r) S[(hg + 4 * r) * kSpRows + key] = valid ? acc[r] : -INFINITY;
  }
  __syncthreads();

  // Per-head softmax statistics of the chunk: warp w takes heads w, w+8, ...
  __shared__ float m_s[kMaxHeads], l_s[kMaxHeads];
  {
    const int lane = tid & 31, w = tid >> 5;
    for (int hd = w; hd < H; hd += kSpThreads / 32) {
      const float x0 = S[hd * kSpRows + lane], x1 = S[hd * kSpRows + lane + 32];
      const float m = warp_max(fmaxf(x0, x1));
      float p0 = 0.f, p1 = 0.f;
      if (m != -INFINITY) {
        p0 = expf(x0 - m);
        p1 = expf(x1 - m);
      }
      const float l = warp_sum(p0 + p1);
      S[hd * kSpRows + lane] = p0;
      S[hd * kSpRows + lane + 32] = p1;
      if (lane == 0) {
        m_s[hd] = m;
        l_s[hd] = l;
      }
    }
  }
  __syncthreads();

  // o[h][d] = sum_r P[h][r] v[r][d]: thread (d = tid % 128, heads tid / 128 + 2k).
  const size_t pidx = (size_t)bq * p.splits4 + split;
  float* po = p.part_o + pidx * H * kHeadDim;
  {
    const int d = tid & (kHeadDim - 1), hg2 = tid >> 7;
#pragma unroll 2
    for (int r = 0; r < H / 2; ++r) {
      const int hd = hg2 + 2 * r;
      const float* pr = S + hd * kSpRows;
      float a = 0.f;
#pragma unroll 8
      for (int j = 0; j < kSpRows; ++j) a = fmaf(pr[j], vs[j * kHeadDim + d], a);
      po[hd * kHeadDim + d] = a;
    }
  }
  for (int hd = tid; hd < H; hd += kSpThreads) {
    p.part_ml[pidx * H * 2 + 2 * hd] = m_s[hd];
    p.part_ml[pidx * H * 2 + 2 * hd + 1] = l_s[hd];
  }
}

template <int H, bool FP8>
static cudaError_t launch_sparse_t(const SparseParams& p, int batch, cudaStream_t st) {
  const size_t smem = sparse_smem_bytes(H);
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(sparse_attn_kernel<H, FP8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  return launch_pdl(sparse_attn_kernel<H, FP8>, dim3(p.splits4, batch * p.n_q), dim3(kSpThreads),
                    smem, st, p);
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
  if (p.chunk4 != kSpRows) return cudaErrorInvalidValue;
  return p.kv.fp8 ? launch_sparse_h<true>(p, batch, st) : launch_sparse_h<false>(p, batch, st);
}

}  // namespace hs2
