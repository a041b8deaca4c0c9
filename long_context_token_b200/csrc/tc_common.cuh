// Shared pieces of the tensor-core (tcgen05) kernels: tile geometry, shared-memory
// layouts of the operands and their descriptors, and host-side TMA tensor maps.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "hs2_internal.cuh"
#include "sm100.cuh"

namespace hs2 {

constexpr int kKeyTile = 128;             // keys per MMA tile (the MMA's M)
constexpr uint32_t kBoxBytes = 16384;     // 128 rows x 64 bf16 (one 128-byte-swizzled box)
constexpr uint32_t kKTileBytesBf16 = 2 * kBoxBytes;  // 128 keys x 128 d x bf16

__host__ __device__ constexpr uint32_t tmem_cols_pow2(int cols) {
  return cols <= 32 ? 32u : cols <= 64 ? 64u : cols <= 128 ? 128u : cols <= 256 ? 256u : 512u;
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Q [H heads][128 d] bf16 -> shared memory as the K-major, unswizzled B operand of
// S^T = K . Q^T: 16-byte chunk c of head h sits at c * (H * 16) + h * 16.
template <int H>
__device__ __forceinline__ void store_q_kmajor(uint8_t* qs, const uint16_t* q, int tid, int nt) {
  for (int e = tid; e < H * (kHeadDim / 8); e += nt) {
    const int h = e % H, c = e / H;
    const uint4 v = *reinterpret_cast<const uint4*>(q + h * kHeadDim + c * 8);
    *reinterpret_cast<uint4*>(qs + c * (H * 16) + h * 16) = v;
  }
}

#ifdef __CUDACC__
// A operand (K tile, K-major, 128-byte swizzle written by TMA): K step kk of 16 d.
__device__ __forceinline__ uint64_t kmajor_sw128_desc(uint32_t tile_addr, int kk) {
  const uint32_t start = tile_addr + (uint32_t)(kk >> 2) * kBoxBytes + (uint32_t)(kk & 3) * 32u;
  return sm100::smem_desc(start, 16, 1024, sm100::kSwizzle128B);
}

// B operand Q (K-major, unswizzled): K step kk covers chunks 2kk and 2kk+1.
template <int H>
__device__ __forceinline__ uint64_t q_kmajor_desc(uint32_t q_addr, int kk) {
  return sm100::smem_desc(q_addr + (uint32_t)kk * 2u * H * 16u, H * 16, 128, sm100::kSwizzleNone);
}

// A operand V^T (V tile is [128 keys][128 d] in two 128-byte-swizzled boxes, so V^T is
// MN-major): K step kk covers keys [16kk, 16kk + 16).
__device__ __forceinline__ uint64_t vt_mnmajor_sw128_desc(uint32_t tile_addr, int kk) {
  return sm100::smem_desc(tile_addr + (uint32_t)kk * 16u * 128u, kBoxBytes, 1024,
                          sm100::kSwizzle128B);
}

// Gather of one tile (index entries [e0, e0 + 128), those at or past e_end absent) into
// the 128-byte-swizzled layout that TMA writes: 16-byte chunk c of row r at box c / 8,
// byte r * 128 + ((c mod 8) xor (r mod 8)) * 16.  K and V rows by cp.async, absent or
// out-of-range entries zero-filled (an out-of-range one also sets the status word).
// The 128 x CHUNKS work items are spread over nthreads threads starting at tid; each
// thread still has to wait for its copies (cp.async.wait_all).  A null kb (vb) skips
// the K (V) rows.
template <int CHUNKS, uint32_t BOX>
__device__ __forceinline__ void gather_tile_rows(uint32_t kdst, uint32_t vdst, const uint8_t* kb,
                                                 const uint8_t* vb, const int32_t* idx_row,
                                                 int e0, int e_end, int Lb, size_t row_base,
                                                 uint32_t* status, int tid, int nthreads) {
  constexpr uint32_t kRowBytes = CHUNKS * 16;
  for (int w = tid; w < kKeyTile * CHUNKS; w += nthreads) {
    const int r = w / CHUNKS, c = w % CHUNKS, e = e0 + r;
    int j = -1;
    if (e < e_end) {
      j = __ldcg(idx_row + e);  // through L2: may have been written by the previous grid
      if (j < 0 || j >= Lb) {
        if (j != -1 && c == 0) set_status(status, HS2_ERR_INDEX_OUT_OF_RANGE);
        j = -1;
      }
    }
    const size_t off = j >= 0 ? (row_base + (size_t)j) * kRowBytes : 0;
    const uint32_t nb = j >= 0 ? 16u : 0u;
    const uint32_t at = (uint32_t)(c >> 3) * BOX + (uint32_t)r * 128u +
                        ((uint32_t)((c & 7) ^ (r & 7)) << 4);
    if (kb) sm100::cp_async_16(kdst + at, kb + off + c * 16, nb);
    if (vb) sm100::cp_async_16(vdst + at, vb + off + c * 16, nb);
  }
}

// Gather of up to 128 rows named by a list in shared memory (rows [0, m) of the tile;
// the rest zero-filled) into the same 128-byte-swizzled layout (K only).  Every listed
// position must lie inside its sequence.  Each thread still has to wait for its copies.
template <int CHUNKS, uint32_t BOX>
__device__ __forceinline__ void gather_list_rows(uint32_t kdst, const uint8_t* kb, const int* list,
                                                 int m, size_t row_base, int tid, int nthreads) {
  constexpr uint32_t kRowBytes = CHUNKS * 16;
  for (int w = tid; w < kKeyTile * CHUNKS; w += nthreads) {
    const int r = w / CHUNKS, c = w % CHUNKS;
    const int j = r < m ? list[r] : -1;
    const size_t off = j >= 0 ? (row_base + (size_t)j) * kRowBytes : 0;
    const uint32_t at = (uint32_t)(c >> 3) * BOX + (uint32_t)r * 128u +
                        ((uint32_t)((c & 7) ^ (r & 7)) << 4);
    sm100::cp_async_16(kdst + at, kb + off + c * 16, j >= 0 ? 16u : 0u);
  }
}

// 2^x with the hardware approximation (relative error about 2^-22), results below the
// normal range flushed to zero; 2^-inf = 0.
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// p0, p1 -> bf16 pairs hi, lo with hi + lo = p to about 16 bits: hi keeps the top 16
// bits of each float (truncation: byte permute), lo = p - hi exactly in float32, then
// rounded to bf16.  Element order as __floats2bfloat162_rn (p0 in the low half).
__device__ __forceinline__ void split_bf16_hi_lo(float p0, float p1, uint32_t& hi, uint32_t& lo) {
  const uint32_t b0 = __float_as_uint(p0), b1 = __float_as_uint(p1);
  hi = __byte_perm(b0, b1, 0x7632);
  const __nv_bfloat162 l2 = __floats2bfloat162_rn(p0 - __uint_as_float(b0 & 0xffff0000u),
                                                  p1 - __uint_as_float(b1 & 0xffff0000u));
  lo = *reinterpret_cast<const uint32_t*>(&l2);
}

// Softmax reference usable in 2^(x - m): a reference of -inf (no key seen yet, so
// every x is -inf too) becomes 0, which gives p = 0 instead of NaN.
__device__ __forceinline__ float finite_ref(float m) { return m == -INFINITY ? 0.f : m; }

// ---- cluster merge of a gathered row (sparse layers)
// Gather-mode CTAs of one row run as a thread-block cluster of ns <= kMaxClusterCtas
// CTAs.  Each leaves its chunk's partial in its own shared memory -- o at offset
// kClusterOOff as [H][128] floats (unnormalised, reference m in log2 units), (m, l)
// at kClusterMlOff as [H][2] floats (l = 0: no key) -- and CTA r then combines heads
// r, r + ns, ... from all ns CTAs through distributed shared memory:
//   out_h = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s,  M = max over non-empty s.
// A row with no key at all gets zeros.  Threads [0, 128) take part (d = thread).
constexpr int kMaxClusterCtas = 16;
constexpr uint32_t kClusterOOff = 0;
constexpr uint32_t kClusterMlOff = 32768;  // o of up to 64 heads fits below

template <int H>
__device__ __forceinline__ void cluster_merge_row(const uint8_t* smem, int ns, float* out_row) {
  static_assert(H * kHeadDim * 4 <= kClusterMlOff, "partial o must fit below (m, l)");
  const int d = threadIdx.x;
  if (d >= kHeadDim) return;
  const uint32_t o_base = sm100::smem_u32(smem + kClusterOOff);
  const uint32_t ml_base = sm100::smem_u32(smem + kClusterMlOff);
  for (int h = (int)sm100::cluster_ctarank(); h < H; h += ns) {
    float m[kMaxClusterCtas], l[kMaxClusterCtas], o[kMaxClusterCtas];
#pragma unroll
    for (int s = 0; s < kMaxClusterCtas; ++s) {
      if (s < ns) {
        const float2 v = sm100::ld_shared_cluster_f32x2(
            sm100::mapa_shared(ml_base + (uint32_t)h * 8u, (uint32_t)s));
        m[s] = v.x;
        l[s] = v.y;
        o[s] = sm100::ld_shared_cluster_f32(
            sm100::mapa_shared(o_base + (uint32_t)(h * kHeadDim + d) * 4u, (uint32_t)s));
      } else {
        m[s] = -INFINITY;
        l[s] = 0.f;
        o[s] = 0.f;
      }
    }
    float M = -INFINITY;
#pragma unroll
    for (int s = 0; s < kMaxClusterCtas; ++s)
      if (l[s] > 0.f) M = fmaxf(M, m[s]);
    float L = 0.f, acc = 0.f;
#pragma unroll
    for (int s = 0; s < kMaxClusterCtas; ++s) {
      if (l[s] > 0.f) {  // an empty partial's o is never read into the sum
        const float w = exp2f(m[s] - M);
        L = fmaf(w, l[s], L);
        acc = fmaf(w, o[s], acc);
      }
    }
    out_row[h * kHeadDim + d] = L > 0.f ? acc / L : 0.f;
  }
}

// B operand P^T (P stored [H/8 chunks][128 keys][8 heads], MN-major, unswizzled):
// K step kk covers keys [16kk, 16kk + 16).
__device__ __forceinline__ uint64_t pt_mnmajor_desc(uint32_t p_addr, int kk) {
  return sm100::smem_desc(p_addr + (uint32_t)kk * 256u, 128, kKeyTile * 16, sm100::kSwizzleNone);
}
#endif

#ifdef __CUDACC__
// ---- E4M3 operands of the kind::f8f6f4 MMAs (FP8 cache)
constexpr uint32_t kE4m3TileBytes = 16384;  // 128 keys x 128 E4M3 codes

// Two floats -> their E4M3 codes (round to nearest even, saturating; y0 in the low
// byte) and the values those codes stand for.
__device__ __forceinline__ uint32_t e4m3_pair(float y0, float y1, float& v0, float& v1) {
  const __nv_fp8x2_storage_t c =
      __nv_cvt_float2_to_fp8x2(make_float2(y0, y1), __NV_SATFINITE, __NV_E4M3);
  const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(c, __NV_E4M3);
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
  v0 = f.x;
  v1 = f.y;
  return (uint32_t)c;
}
__device__ __forceinline__ uint32_t e4m3_codes(float y0, float y1) {
  return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(y0, y1), __NV_SATFINITE, __NV_E4M3);
}

// Q [H][128] bf16 -> the B operand of S^T = K . [Q_hi | Q_lo]^T (K-major, unswizzled,
// N = 2H rows: row h holds Q_hi of head h, row H + h its Q_lo): 16-byte chunk c (16 d)
// of row n at c * (2H * 16) + n * 16.  y = q * 2^e with the largest |y| in [128, 256),
// Q_hi = E4M3(y), Q_lo = E4M3(16 (y - Q_hi)) (y - Q_hi is exact in float32).
// *qinv = 2^-e.  Every thread of the block calls this; it ends with __syncthreads.
template <int H>
__device__ void store_q_e4m3_split(uint8_t* qs, const uint16_t* qg, float* qinv) {
  __shared__ float hmax_s[kMaxHeads];
  __shared__ float up_s;
  const int warp = threadIdx.x >> 5, nw = blockDim.x >> 5, lane = threadIdx.x & 31;
  for (int h = warp; h < H; h += nw) {
    float m = 0.f;
    for (int c = lane; c < kHeadDim; c += 32)
      m = fmaxf(m, fabsf(__uint_as_float((uint32_t)qg[h * kHeadDim + c] << 16)));
    m = warp_max(m);
    if (lane == 0) hmax_s[h] = m;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = 0.f;
    for (int h = 0; h < H; ++h) m = fmaxf(m, hmax_s[h]);
    int e = 0;
    if (m > 0.f) {
      int ex;
      frexpf(m, &ex);  // m in [2^(ex-1), 2^ex)
      e = 8 - ex;
      e = e < -100 ? -100 : (e > 100 ? 100 : e);
    }
    up_s = __int_as_float((127 + e) << 23);
    *qinv = __int_as_float((127 - e) << 23);
  }
  __syncthreads();
  const float sc = up_s;
  for (int w = threadIdx.x; w < H * (kHeadDim / 16); w += blockDim.x) {
    const int h = w % H, c = w / H;
    const uint4 a = *reinterpret_cast<const uint4*>(qg + h * kHeadDim + c * 16);
    const uint4 b = *reinterpret_cast<const uint4*>(qg + h * kHeadDim + c * 16 + 8);
    const uint32_t in[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      hi[u] = 0u;
      lo[u] = 0u;
#pragma unroll
      for (int v = 0; v < 2; ++v) {
        const uint32_t x = in[2 * u + v];
        const float y0 = __uint_as_float(x << 16) * sc;
        const float y1 = __uint_as_float(x & 0xffff0000u) * sc;
        float a0, a1;
        const uint32_t ch = e4m3_pair(y0, y1, a0, a1);
        const uint32_t cl = e4m3_codes((y0 - a0) * 16.f, (y1 - a1) * 16.f);
        hi[u] |= ch << (16 * v);
        lo[u] |= cl << (16 * v);
      }
    }
    *reinterpret_cast<uint4*>(qs + c * (2 * H * 16) + h * 16) =
        make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(qs + c * (2 * H * 16) + (H + h) * 16) =
        make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
  __syncthreads();
}

// A operand K (K-major, 128-byte swizzle, one 128-byte row per key): K step kk of 32 d.
__device__ __forceinline__ uint64_t k_e4m3_desc(uint32_t tile, int kk) {
  return sm100::smem_desc(tile + (uint32_t)kk * 32u, 16, 1024, sm100::kSwizzle128B);
}
// B operand [Q_hi | Q_lo] (K-major, unswizzled, N rows): K step kk of 32 d.
template <int N>
__device__ __forceinline__ uint64_t q_e4m3_desc(uint32_t q, int kk) {
  return sm100::smem_desc(q + (uint32_t)kk * 2u * N * 16u, N * 16, 128, sm100::kSwizzleNone);
}
// A operand V^T: the V tile is [128 keys][128 codes] with 128-byte swizzle, so V^T is
// MN-major with all 128 d inside one swizzle atom; K step kk of 32 keys (four atoms
// of 8 keys, 1024 bytes apart).
__device__ __forceinline__ uint64_t vt_e4m3_desc(uint32_t tile, int kk) {
  return sm100::smem_desc(tile + (uint32_t)kk * 32u * 128u, kE4m3TileBytes, 1024,
                          sm100::kSwizzle128B);
}
// B operand P^T: P stored [3H / 16 chunks][128 keys][16 codes] (MN-major, unswizzled;
// chunk (term * H + h) / 16 holds heads h..h+15 of one term); K step kk of 32 keys.
__device__ __forceinline__ uint64_t pt_e4m3_desc(uint32_t p, int kk) {
  return sm100::smem_desc(p + (uint32_t)kk * 32u * 16u, 128, kKeyTile * 16, sm100::kSwizzleNone);
}

#endif

// Host: 2-D tiled tensor map over a row-major [rows][inner] array.
bool make_tmap_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t inner,
                  uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows,
                  CUtensorMapSwizzle swizzle);

cudaError_t launch_full_attn_tc(const FullParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                                int bq, cudaStream_t st);
// Sparse layer through the same kernel in gather mode (p.idx, p.idx_width, p.out set):
// one thread-block cluster per row merges its chunks on chip; the launcher chooses
// p.splits1 (the cluster size) and p.chunk1.
cudaError_t launch_sparse_attn_tc(FullParams p, int bq, cudaStream_t st);
// The same two kernels for an FP8 E4M3 cache (tensor maps over uint8 rows).
cudaError_t launch_full_attn_fp8(const FullParams& p, const CUtensorMap& tk,
                                 const CUtensorMap& tv, int bq, cudaStream_t st);
cudaError_t launch_sparse_attn_fp8(FullParams p, int bq, cudaStream_t st);
// Chunking of a gathered row over a cluster of at most max_ctas CTAs: chunks of whole
// 128-entry tiles, as many CTAs as tiles while they fit.
void plan_gather_cluster(int idx_width, int max_ctas, int* ns, int* chunk);
// Largest cluster size (16, 8, 4, 2 or 1; 0 if none) with which one cluster of the
// kernel can be resident, given its block size and dynamic shared memory.
int largest_cluster_of(const void* kernel, dim3 block, size_t smem);
template <typename K>
int largest_cluster(K* kernel, dim3 block, size_t smem) {
  return largest_cluster_of(reinterpret_cast<const void*>(kernel), block, smem);
}
// Full layer for several new tokens per sequence (or 128 heads), bf16 cache: 128 query
// rows (G = 128 / h tokens x h heads) per CTA, 64-key tiles (tensor maps with 64 x 64
// boxes).  Partials in the one-token kernel's layout.
cudaError_t launch_full_attn_mq(const FullParams& p, const CUtensorMap& tk,
                                const CUtensorMap& tv, int batch, cudaStream_t st);
int mq_tokens_per_cta(int h);
inline bool mq_eligible(int n_q, int h) {
  return (h == 16 || h == 32 || h == 48 || h == 64 || h == 128) && (n_q >= 2 || h > 64);
}
cudaError_t launch_importance_tc(const SelectParams& p, const CUtensorMap& tmap_k, int bq,
                                 cudaStream_t st);
// Importance pass for the several-token shapes (bf16): G = 128 / h tokens per CTA;
// p.chunk2 a multiple of 128 below 65536.
cudaError_t launch_importance_mq(const SelectParams& p, const CUtensorMap& tmap_k, int batch,
                                 cudaStream_t st);
cudaError_t launch_importance_fp8(const SelectParams& p, const CUtensorMap& tmap_k, int bq,
                                  cudaStream_t st);

}  // namespace hs2
