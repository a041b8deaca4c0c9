// Full-attention layer (and, in gather mode, a reusing sparse layer) on the
// 5th-generation tensor cores for an FP8 E4M3 KV cache with per-token scales
// (web coverage of HySparse2: the 1M-token footprint is quoted with an FP8 KV cache;
// "Luo Fuli Teases Xiaomi MiMo-V3 Architecture ...", paragraph on cost at 1M tokens).
//
// The cache's E4M3 codes feed the MMA as they are (kind::f8f6f4, both operands E4M3,
// fp32 accumulation), straight from the tiles TMA writes; the per-token scales stay
// out of it: k_scale[j] multiplies key j's logits and v_scale[j] its probability
// before P.V.  The other two operands are sums of E4M3 terms:
//   Q = 2^-e (Q_hi + Q_lo / 16), one power of two for all heads putting the largest
//     |q| into [128, 256): a bf16 element (8 significant bits) whose scaled magnitude
//     is at least 2^-6 is exact in the two terms, smaller ones to 2^-13 absolute;
//   P' = p * v_scale * 2^-ev rounded to f16 (11 significant bits, as an f16 P would
//     carry) = P_hi + P_lo / 16 + P_lo2 / 256 (exact for P' >= 2^-6; below, within
//     2^-18 absolute, 2^-26 of the largest P' of 256), ev a power of two at or above
//     every |v_scale| the CTA has seen, moved with a rescale of O (like the softmax
//     reference) when a larger one arrives.
// So S^T [128 keys x 2H] = K . [Q_hi | Q_lo]^T and O^T [128 d x 3H] += V^T . [P_hi |
// P_lo | P_lo2]^T; the softmax and the epilogue combine each head's columns.
//
// One CTA per key chunk (or per 128 index entries) of one (sequence, token):
//   warp 0      producer: TMA of 128-row E4M3 tiles (128-byte rows, 128-byte
//               swizzle) into an R-stage ring, K and V on their own barriers; in
//               gather mode cp.async of the indexed rows into the same layout;
//   warp 1      TMEM allocator and MMA issuer: K (K-major) and V^T (MN-major) are
//               read from the ring, whose stages the MMA commits release;
//   warps 2..   softmax: one key per thread (two threads per key at 64 heads, 32
//               heads each), lazily moved per-head reference, P written as its three
//               E4M3 terms.
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <string.h>

#include "hs2_internal.cuh"
#include "sm100.cuh"
#include "tc_common.cuh"
#include "decode_select.cuh"

namespace hs2 {

using namespace sm100;

namespace {

constexpr float kLog2eF8 = 1.4426950408889634f;
constexpr float kRescaleAtF8 = 8.0f;
constexpr int kNoScale = -1000;  // exponent of a CTA that has seen no V scale yet
// Softmax threads per key: two at 64 heads (each takes 32 of the key's heads, so that
// its logits, references and running sums stay in registers), else one.
template <int H>
__host__ __device__ constexpr int fp8_halves() { return H == 64 ? 2 : 1; }
template <int H>
__host__ __device__ constexpr int fp8_threads() { return 64 + 128 * fp8_halves<H>(); }
constexpr uint32_t kRawTile = 16384;    // 128 keys x 128 E4M3 codes

template <int H, bool GATHER>
struct Fp8Smem {
  static constexpr uint32_t kQBytes = 2 * H * kHeadDim;       // Q_hi, Q_lo rows
  static constexpr uint32_t kPBytes = 3 * H * kKeyTile;       // P_hi, P_lo, P_lo2
  static constexpr uint32_t kRedBytes = (4 * H + 8) * 4;      // [4 warps][H] + V-scale maxima
  static constexpr uint32_t kRefBytes = (2 * H + 8) * 4;      // mref, alpha, scalars
  static constexpr uint32_t kMaxBars = 4 * 6 + 10 + kTileRing;
  // Full layer only: the histogram of the selection bounds u and the exchange of the two
  // head halves' partial bounds ([2][128] floats).
  static constexpr uint32_t kSelBytes = GATHER ? 0u : kUHistBytes + 2u * 128u * 4u;
  // (+ 1024 for alignment, + 1024 for the static shared memory of the Q staging, + 7168
  // for that of the fused tail)
  static constexpr uint32_t kFixed = kQBytes + 2 * kPBytes + kRedBytes + kRefBytes +
                                     kMaxBars * 8 + 16 + 4 * kTileRing + kSelBytes + 2048 +
                                     (GATHER ? 0 : 7168);
  // Raw stages (K and V each): as many as fit, up to six; gather mode keeps one (its
  // CTAs mostly take a single tile).
  static constexpr int kFit = (int)((227u * 1024u - kFixed) / (2 * kRawTile));
  static constexpr int R = GATHER ? 1 : (kFit > 6 ? 6 : kFit);
  static constexpr uint32_t kKRawOff = 0;
  static constexpr uint32_t kVRawOff = R * kRawTile;
  static constexpr uint32_t kQOff = 2 * R * kRawTile;
  static constexpr uint32_t kPOff = kQOff + kQBytes;          // [2 buffers]
  static constexpr uint32_t kRedOff = kPOff + 2 * kPBytes;
  static constexpr uint32_t kRefOff = kRedOff + kRedBytes;
  static constexpr uint32_t kBarOff = kRefOff + kRefBytes;
  static constexpr uint32_t kBars = 4 * R + 10 + kTileRing;
  static constexpr uint32_t kSlotOff = kBarOff + kBars * 8;
  static constexpr uint32_t kRingOff = kSlotOff + 16;  // [kTileRing] tile indices
  static constexpr uint32_t kUHistOff = (kRingOff + 4 * kTileRing + 15) / 16 * 16;
  static constexpr uint32_t kUxOff = kUHistOff + (GATHER ? 0u : kUHistBytes);
  static constexpr uint32_t kBytes = kUHistOff + kSelBytes + 1024;
  static constexpr uint32_t kTmemCols = tmem_cols_pow2(7 * H);  // S: 2 x 2H, O: 3H
  static_assert(R >= 1 && kBytes <= 227 * 1024, "shared memory budget");
  static_assert(kQOff + kQBytes >= kClusterMlOff + 2 * H * 4, "cluster partial fits");
  static_assert(kQOff % 1024 == 0 && kPOff % 16 == 0 && kBarOff % 8 == 0, "alignment");
};

// Two f16 values y (11 significant bits, |y| <= 448) -> three pairs of E4M3 codes with
// y = hi + lo / 16 + lo2 / 256 (4 + 4 + 3 bits; every difference and scaling below is
// exact in f16): exactly for |y| >= 2^-6, to 2^-18 absolute below (E4M3 subnormals).
// Element 0 in the low byte of each pair.
__device__ __forceinline__ void e4m3_split3(__half2 y, uint32_t& hi, uint32_t& lo, uint32_t& lo2) {
  const __half2 k16 = __float2half2_rn(16.f);
  hi = (uint32_t)__nv_cvt_halfraw2_to_fp8x2(y, __NV_SATFINITE, __NV_E4M3);
  const __half2 a = __half2(__nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)hi, __NV_E4M3));
  const __half2 r = __hmul2(__hsub2(y, a), k16);
  lo = (uint32_t)__nv_cvt_halfraw2_to_fp8x2(r, __NV_SATFINITE, __NV_E4M3);
  const __half2 b = __half2(__nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)lo, __NV_E4M3));
  lo2 = (uint32_t)__nv_cvt_halfraw2_to_fp8x2(__hmul2(__hsub2(r, b), k16), __NV_SATFINITE,
                                             __NV_E4M3);
}

// Named barrier of head group `half` over its 128 threads, with compile-time ids (1, 2)
// so that the kernel reserves only the barriers it names.
__device__ __forceinline__ void group_bar_sync(int half) {
  if (half) sm100::named_bar_sync(2, 128);
  else sm100::named_bar_sync(1, 128);
}
__device__ __forceinline__ bool group_bar_or(int half, bool pred) {
  return half ? sm100::named_bar_or(5, 128, pred) : sm100::named_bar_or(4, 128, pred);
}

// Largest value over the 128 softmax threads of one head group (heads [hoff, hoff + HH)),
// per head (the group's named barrier).
template <int HH, int H>
__device__ __forceinline__ void block_max_group_f8(const float (&v)[HH], float* red, float* out,
                                                   int t, int hoff, int half) {
  const int w = t >> 5, lane = t & 31;
#pragma unroll
  for (int h = 0; h < HH; ++h) {
    const float m = warp_max(v[h]);
    if (lane == 0) red[w * H + hoff + h] = m;
  }
  group_bar_sync(half);
  if (t < HH)
    out[hoff + t] = fmaxf(fmaxf(red[hoff + t], red[H + hoff + t]),
                          fmaxf(red[2 * H + hoff + t], red[3 * H + hoff + t]));
  group_bar_sync(half);
}

}  // namespace

// Fused tail of the full layer, as in the bf16 kernel (decode_select.cuh): a function of
// its own whose indices are recomputed from the CTA's coordinates.  The candidates' E4M3 K
// rows go through the stream's own kind::f8f6f4 MMA against [Q_hi | Q_lo] (S buffers of 2H
// columns), and at 64 heads the two head halves combine their partial keys through ux_s.
// The float64 re-scoring reads the bf16 query from global memory.
template <int H>
__device__ __noinline__ bool full_fp8_tail(const FullParams& p) {
  using L = Fp8Smem<H, false>;
  constexpr int R = L::R;
  constexpr int NHALF = fp8_halves<H>();
  constexpr int HH = H / NHALF;
  constexpr int NSOFT = 128 * NHALF;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t k_addr = smem_u32(smem + L::kKRawOff);
  const uint32_t q_addr = smem_u32(smem + L::kQOff);
  const float* qsc_s = reinterpret_cast<const float*>(smem + L::kRefOff) + 2 * H;
  uint64_t* post_bar = reinterpret_cast<uint64_t*>(smem + L::kBarOff) + 4 * R + 9;
  const uint32_t* tmem_slot = reinterpret_cast<const uint32_t*>(smem + L::kSlotOff);
  const uint32_t* uhist_s = reinterpret_cast<const uint32_t*>(smem + L::kUHistOff);
  float* ux_s = reinterpret_cast<float*>(smem + L::kUxOff);
  const int warp = threadIdx.x >> 5;
  const int split = blockIdx.x, bq = blockIdx.y;
  const int b = bq / p.n_q, qi = bq % p.n_q;
  const int pos = seq_len(p.kv, b, p.n_q, p.status, false) - p.n_q + qi;
  const int k0 = split * p.chunk1;
  const int k1 = min(k0 + p.chunk1, pos + 1);
  const size_t row_base = (size_t)b * p.kv.max_len;
  const float c2 = p.sm_scale * kLog2eF8 * qsc_s[0];
  auto recompute = [&](const int* list, int m, float* t2, uint32_t round, const float* D) -> bool {
    bool rok = true;
    const int ntile = (m + kKeyTile - 1) / kKeyTile;
    for (int tl = 0; tl < ntile; ++tl)
      gather_list_rows<8, kRawTile>(k_addr + tl * kRawTile, static_cast<const uint8_t*>(p.kv.k),
                                    list + tl * kKeyTile, min(kKeyTile, m - tl * kKeyTile),
                                    row_base, threadIdx.x, blockDim.x);
    cp_async_wait_all();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    if (warp == 1) {
      if (elect_one()) {
        constexpr uint32_t id_qk = idesc_e4m3(128, 2 * H, false, false);
        for (int tl = 0; tl < ntile; ++tl) {
#pragma unroll
          for (int kk = 0; kk < kHeadDim / 32; ++kk)
            mma_e4m3_ss(tmem_base + tl * 2 * H, k_e4m3_desc(k_addr + tl * kRawTile, kk),
                        q_e4m3_desc<2 * H>(q_addr, kk), id_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(post_bar);
      }
      __syncwarp();
    } else if (warp >= 2) {
      const int lg = warp & 3;
      const int t = lg * 32 + (int)lane_id();
      const int half = (warp - 2) >> 2;
      const int hoff = half * HH;
      const uint32_t lane_base = (uint32_t)(lg * 32) << 16;
      if (!mbar_wait(post_bar, round & 1u)) rok = false;
      tc_fence_after();
      for (int tl = 0; tl < ntile; ++tl) {
        uint32_t r[2 * HH];
#pragma unroll
        for (int c = 0; c < HH; c += 16) {
          tmem_ld16(tmem_base + lane_base + tl * 2 * H + hoff + c,
                    *reinterpret_cast<uint32_t(*)[16]>(r + c));
          tmem_ld16(tmem_base + lane_base + tl * 2 * H + H + hoff + c,
                    *reinterpret_cast<uint32_t(*)[16]>(r + HH + c));
        }
        tmem_wait_ld();
        const int slot = tl * kKeyTile + t;
        const int jj = slot < m ? list[slot] : -1;
        const float cks = jj >= 0 ? c2 * __ldg(p.kv.k_scale + row_base + jj) : 0.f;
        float v = -INFINITY;
#pragma unroll
        for (int e = 0; e < HH; ++e)
          v = fmaxf(v, fmaf(__uint_as_float(r[HH + e]), 0.0625f, __uint_as_float(r[e])) * cks -
                           D[hoff + e]);
        if (NHALF == 2) {
          if (half == 1) ux_s[t] = v;
          named_bar_sync(3, NSOFT);
          if (half == 0) v = fmaxf(v, ux_s[t]);
          named_bar_sync(3, NSOFT);  // ux_s is reused by the next tile
        }
        if (half == 0 && jj >= 0) t2[slot] = v;
      }
      tc_fence_before();
    }
    __syncthreads();
    return rok;
  };
  QView qv;
  qv.base = reinterpret_cast<const uint8_t*>(p.q + (size_t)bq * H * kHeadDim);
  qv.hstride = kHeadDim * 2;  // bf16 rows [H][128] in global memory
  qv.cstride = 16;
  // The partial's m per head is still in the softmax warps' reference array, unless the
  // CTA took no tile (the same rule as the stream's).
  const bool dyn = p.splits1 > 1 && !p.deterministic;
  const bool took = dyn ? split < (pos + kKeyTile) / kKeyTile : k0 < k1;
  const float* own_m = took ? reinterpret_cast<const float*>(smem + L::kRefOff) : nullptr;
  return fused_tail<H, true, fp8_threads<H>() / 32>(p, smem, 2u * R * kRawTile, kRawTile, uhist_s,
                                                     own_m, bq, b, split, pos, k0, k1, qv,
                                                     recompute);
}

template <int H, bool GATHER>
__global__ void __launch_bounds__(fp8_threads<H>(), 1)
    full_attn_fp8_kernel(const __grid_constant__ CUtensorMap tmap_k,
                         const __grid_constant__ CUtensorMap tmap_v,
                         const __grid_constant__ FullParams p) {
  using L = Fp8Smem<H, GATHER>;
  constexpr int R = L::R;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* kraw = smem + L::kKRawOff;
  uint8_t* vraw = smem + L::kVRawOff;
  uint8_t* qs = smem + L::kQOff;
  uint8_t* ps = smem + L::kPOff;
  float* red = reinterpret_cast<float*>(smem + L::kRedOff);  // [4][H], then [2 groups][4]
  float* mref_s = reinterpret_cast<float*>(smem + L::kRefOff);
  float* alpha_s = mref_s + H;
  float* qsc_s = mref_s + 2 * H;  // [0]: 2^-e of Q
  int* ev_s = reinterpret_cast<int*>(mref_s + 2 * H + 2);    // [2 groups]
  float* beta_s = mref_s + 2 * H + 4;                         // [2 groups]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* kr_full = bars;
  uint64_t* kr_empty = bars + R;
  uint64_t* vr_full = bars + 2 * R;
  uint64_t* vr_empty = bars + 3 * R;
  uint64_t* s_full = bars + 4 * R;  // [2]
  uint64_t* s_free = s_full + 2;    // [2]
  uint64_t* p_full = s_full + 4;    // [2]
  uint64_t* p_free = s_full + 6;    // [2]
  uint64_t* mma_done = s_full + 8;
  uint64_t* post_bar = s_full + 9;  // MMAs of the selection tail
  uint64_t* idx_bar = s_full + 10;  // [kTileRing] one per slot of the tile-index ring
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kSlotOff);
  int* tile_ring = reinterpret_cast<int*>(smem + L::kRingOff);
  uint32_t* uhist_s = reinterpret_cast<uint32_t*>(smem + L::kUHistOff);
  float* ux_s = reinterpret_cast<float*>(smem + L::kUxOff);  // [2][128]

  const int warp = threadIdx.x >> 5;
  const int split = blockIdx.x, bq = blockIdx.y;
  const int b = bq / p.n_q, qi = bq % p.n_q;

  // Set-up that touches no global memory, overlapping the previous kernel's tail.
  if (threadIdx.x == 0) {
    for (int s = 0; s < R; ++s) {
      mbar_init(kr_full + s, GATHER ? 32 : 1);
      mbar_init(kr_empty + s, 1);
      mbar_init(vr_full + s, GATHER ? 32 : 1);
      mbar_init(vr_empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(s_full + s, 1);
      mbar_init(s_free + s, 128 * fp8_halves<H>());
      mbar_init(p_full + s, 128 * fp8_halves<H>());
      mbar_init(p_free + s, 1);
      ev_s[s] = kNoScale;
      beta_s[s] = 0.f;
    }
    mbar_init(mma_done, 1);
    mbar_init(post_bar, 1);
    for (int r = 0; r < kTileRing; ++r) mbar_init(idx_bar + r, 1);
    fence_mbar_init();
  }
  if (!GATHER)
    for (int e = threadIdx.x; e < kUBins; e += blockDim.x) uhist_s[e] = 0u;
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  if (!GATHER && warp == 0 && lane_id() == 0) {
    prefetch_tmap(&tmap_k);
    prefetch_tmap(&tmap_v);
  }
  // A sparse layer waits for the previous grid only before writing its output (see the
  // bf16 kernel: nothing it reads is written by the previous kernel of this library).
  const bool defer_wait = GATHER && p.out != nullptr;
  if (!defer_wait) griddep_wait();
  // A sparse layer lets the next kernel start at once: the next sparse layer needs
  // nothing from this one and, like this one, waits before writing its output; every
  // other kernel of the library waits for this grid to end before it reads anything.
  if (defer_wait) griddep_launch_dependents();

  const int Lb = seq_len(p.kv, b, p.n_q, p.status, !GATHER && split == 0 && qi == 0);
  const int pos = Lb - p.n_q + qi;
  const int k0 = split * p.chunk1;
  const int k1 = GATHER ? min(k0 + p.chunk1, p.idx_width) : min(k0 + p.chunk1, pos + 1);
  const int32_t* idx_row = GATHER ? p.idx + (size_t)bq * p.idx_width : nullptr;
  const size_t row_base = (size_t)b * p.kv.max_len;
  // Fused full layer with several CTAs a row: the row's tiles are shared out at run time
  // (CTA r takes tiles r, r + S, ..., r + (R - 1) S, then claims the next free tile from
  // the row's counter), as in the bf16 kernel; the selection keeps its static chunks.
  const int S = p.splits1;
  const bool dyn = !GATHER && p.fuse != 0 && S > 1 && !p.deterministic;
  const int row_tiles = (pos + 1 + kKeyTile - 1) / kKeyTile;
  const int n_tiles = dyn ? (split < row_tiles ? 1 : 0)  // (only whether any)
                          : (k0 < k1 ? (k1 - k0 + kKeyTile - 1) / kKeyTile : 0);
  const int k_end = dyn ? pos + 1 : k1;  // entries at or past this one are absent
  const size_t pidx = (size_t)bq * p.splits1 + split;

  // Row of the cache behind tile entry e (or -1 for an absent / past-the-end entry).
  auto entry_row = [&](int e) -> long long {
    if (e < 0 || e >= k_end) return -1;
    if (!GATHER) return (long long)(row_base + e);
    const int j = __ldcg(idx_row + e);  // through L2: may have been written by the previous grid
    return (j >= 0 && j < Lb) ? (long long)(row_base + j) : -1;
  };
  bool ok = true;
  // Cluster mode keeps the partial in this CTA's shared memory (the raw stages and the
  // Q operand, idle by the time the partial is written) for the on-chip merge.
  const bool on_chip = GATHER && p.out != nullptr;
  float* part_o = on_chip ? reinterpret_cast<float*>(smem + kClusterOOff)
                          : p.part_o + pidx * H * kHeadDim;
  float* part_ml = on_chip ? reinterpret_cast<float*>(smem + kClusterMlOff)
                           : p.part_ml + pidx * H * 2;

  if (n_tiles == 0) {
    for (int h = threadIdx.x; h < H; h += blockDim.x) {
      part_ml[2 * h] = -INFINITY;
      part_ml[2 * h + 1] = 0.f;
    }
  } else {
  if (GATHER) {
    // The first tile's rows are gathered by every thread of the CTA (absent entries
    // zero-filled); warp 0 gathers any later tiles.  (store_q_e4m3_split below
    // synchronises the block.)
    gather_tile_rows<8, kRawTile>(smem_u32(kraw), smem_u32(vraw),
                                  static_cast<const uint8_t*>(p.kv.k),
                                  static_cast<const uint8_t*>(p.kv.v), idx_row, k0, k1, Lb,
                                  row_base, p.status, threadIdx.x, blockDim.x);
  }
  store_q_e4m3_split<H>(qs, p.q + (size_t)bq * H * kHeadDim, qsc_s);
  if (GATHER) cp_async_wait_all();
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t tmem_o = tmem_base + 4 * H;

  if (warp == 0) {
    if (GATHER) {
      // ---------------------------------------------- gather producer (32 lanes)
      const int lane = (int)lane_id();
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i % R;
        if (i == 0) {  // tile 0 was gathered by the whole CTA above
          mbar_arrive(kr_full + s);
          mbar_arrive(vr_full + s);
          continue;
        }
        // K and V separately, each once its stage is released: with one stage, V's is
        // released by P.V of the previous tile, which the MMA issues only after this
        // tile's Q.K^T.
        const uint32_t ph = ((i / R) & 1) ^ 1;
        const int e0 = k0 + i * kKeyTile;
        if (ok && !mbar_wait(kr_empty + s, ph)) ok = false;
        gather_tile_rows<8, kRawTile>(smem_u32(kraw + s * kRawTile), 0,
                                      static_cast<const uint8_t*>(p.kv.k), nullptr, idx_row, e0,
                                      k1, Lb, row_base, p.status, lane, 32);
        cp_async_wait_all();
        fence_proxy_async_smem();
        mbar_arrive(kr_full + s);
        if (ok && !mbar_wait(vr_empty + s, ph)) ok = false;
        gather_tile_rows<8, kRawTile>(0, smem_u32(vraw + s * kRawTile), nullptr,
                                      static_cast<const uint8_t*>(p.kv.v), idx_row, e0, k1, Lb,
                                      row_base, p.status, lane, 32);
        cp_async_wait_all();
        fence_proxy_async_smem();
        mbar_arrive(vr_full + s);
      }
    } else if (elect_one()) {
      // ---------------------------------------------------------- TMA producer
      // Tile i's index goes to slot i of the ring (its barrier arrived on) before the
      // tile's loads; past the last tile an index of -1 ends the other warps' loops.
      const uint64_t pol = policy_evict_first();
      const int row_b = b * p.kv.max_len;
      uint32_t* row_counter = p.rowsync + (size_t)bq * 8 + kRowTileSlot;
      uint32_t claimed = 0;
      int issued = 0;
      for (int i = 0; ok; ++i) {
        const int s = i % R;
        const uint32_t ph = ((i / R) & 1) ^ 1;
        const int tile = dyn ? (i < R ? split + i * S : R * S + (int)claimed)
                             : (i < n_tiles ? k0 / kKeyTile + i : -1);
        const bool end = tile < 0 || tile >= row_tiles || (!dyn && i >= n_tiles);
        if (!mbar_wait(kr_empty + s, ph)) { ok = false; break; }
        tile_ring[i % kTileRing] = end ? -1 : tile;
        mbar_arrive(idx_bar + i % kTileRing);
        if (end) break;
        if (dyn && i + 1 >= R) claimed = atomicAdd(row_counter, 1u);  // tile i + 1's
        const int row = row_b + tile * kKeyTile;
        mbar_arrive_expect_tx(kr_full + s, kRawTile);
        tma_load_2d(kraw + s * kRawTile, &tmap_k, kr_full + s, 0, row, pol);
        if (!mbar_wait(vr_empty + s, ph)) { ok = false; break; }
        mbar_arrive_expect_tx(vr_full + s, kRawTile);
        tma_load_2d(vraw + s * kRawTile, &tmap_v, vr_full + s, 0, row, pol);
        issued = i + 1;
      }
      for (int i = issued > R ? issued - R : 0; i < issued; ++i) {
        if (!mbar_wait(kr_full + (i % R), (i / R) & 1)) ok = false;
        if (!mbar_wait(vr_full + (i % R), (i / R) & 1)) ok = false;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      constexpr uint32_t id_qk = idesc_e4m3(128, 2 * H, false, false);
      constexpr uint32_t id_pv = idesc_e4m3(128, 3 * H, true, true);
      const uint32_t q_addr = smem_u32(qs);
      auto issue_pv = [&](int t) -> bool {
        const int s = t % R, pb = t & 1;
        if (!mbar_wait(vr_full + s, (t / R) & 1)) return false;
        if (!mbar_wait(p_full + pb, (t >> 1) & 1)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(vraw + s * kRawTile);
        const uint32_t p_addr = smem_u32(ps + pb * L::kPBytes);
#pragma unroll
        for (int kk = 0; kk < kKeyTile / 32; ++kk)
          mma_e4m3_ss(tmem_o, vt_e4m3_desc(v_addr, kk), pt_e4m3_desc(p_addr, kk), id_pv,
                      (t > 0 || kk > 0) ? 1u : 0u);
        mma_commit(p_free + pb);
        mma_commit(vr_empty + s);
        return true;
      };
      int n_done = 0;
      for (int i = 0; (GATHER ? i < n_tiles : true) && ok; ++i) {
        const int s = i % R, sb = i & 1;
        if (!GATHER) {  // the tile's index first (-1: past the last tile)
          if (!mbar_wait(idx_bar + i % kTileRing, (i / kTileRing) & 1)) { ok = false; break; }
          if (tile_ring[i % kTileRing] < 0) break;
        }
        if (!mbar_wait(kr_full + s, (i / R) & 1)) { ok = false; break; }
        n_done = i + 1;
        if (!mbar_wait(s_free + sb, ((i >> 1) & 1) ^ 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(kraw + s * kRawTile);
#pragma unroll
        for (int kk = 0; kk < kHeadDim / 32; ++kk)
          mma_e4m3_ss(tmem_base + sb * 2 * H, k_e4m3_desc(k_addr, kk),
                      q_e4m3_desc<2 * H>(q_addr, kk), id_qk, kk > 0 ? 1u : 0u);
        mma_commit(s_full + sb);
        mma_commit(kr_empty + s);
        if (i > 0 && !issue_pv(i - 1)) { ok = false; break; }
      }
      if (ok && n_done > 0 && !issue_pv(n_done - 1)) ok = false;
      mma_commit(mma_done);
      if (!mbar_wait(mma_done, 0)) ok = false;
    }
  } else {
    // ------------------------------------------------------------ softmax
    // Thread (t, half): key t of the tile (TMEM lane t), heads [hoff, hoff + HH).
    constexpr int NHALF = fp8_halves<H>();
    constexpr int HH = H / NHALF;
    constexpr int NSOFT = 128 * NHALF;
    const int lg = warp & 3;
    const int t = lg * 32 + (int)lane_id();
    const int half = (warp - 2) >> 2;
    const int hoff = half * HH;
    const uint32_t lane_base = (uint32_t)(lg * 32) << 16;
    const uint64_t keep_policy = policy_evict_last();
    // Fused selection: keys [0, n_c) record their bound u_j = max_h x_hj and count it.  At
    // 64 heads the two halves' partial maxima meet in ux_s one tile later (after the
    // next tile's barrier 3), and half 0 records them.
    const int n_c = pos - p.window + 1;
    const bool sel_keys = !GATHER && p.fuse == 2 && n_c > p.k_sel;
    float* urow = sel_keys ? p.ubuf + (size_t)bq * p.ld_u : nullptr;
    float u_prev = -INFINITY;
    int j_prev = 0;
    bool rec_prev = false;
    auto record_u = [&](int jj, float u) {
      st_global_f32_hint(urow + jj, u, keep_policy);
      atomicAdd(&uhist_s[ubin(u)], 1u);
    };
    // This group's references: in registers up to 16 heads per thread; above, read
    // from shared memory at each use (registers are the limit there).
    constexpr bool kRefRegs = HH <= 16;
    float l[HH], mr[kRefRegs ? HH : 1];
#pragma unroll
    for (int h = 0; h < HH; ++h) {
      l[h] = 0.f;
      if (kRefRegs) mr[kRefRegs ? h : 0] = -INFINITY;
    }
    auto ref = [&](int h) { return kRefRegs ? mr[kRefRegs ? h : 0] : mref_s[hoff + h]; };
    if (t < HH) mref_s[hoff + t] = -INFINITY;
    group_bar_sync(half);
    // V scales: |v_scale| <= vlim = 2^ev for every key seen; P' = p * v_scale * 2^-ev.
    int ev = kNoScale;
    float vlim = 0.f, vmul = 0.f;
    // Per-key scales (and validity) are loaded two tiles ahead so that their memory
    // latency overlaps the tiles in between instead of stalling each tile.
    // Tiles in the order this CTA takes them, by their first entry: k0 + 128 i in gather
    // mode, else from the producer's ring (read in order, never past its -1).
    int seen = 0;
    bool ring_end = false;
    auto next_base = [&]() -> int {
      int v = -1;
      if (GATHER) {
        v = seen < n_tiles ? k0 + seen * kKeyTile : -1;
      } else if (!ring_end) {
        if (ok && !mbar_wait(idx_bar + seen % kTileRing, (seen / kTileRing) & 1)) ok = false;
        const int tl = ok ? tile_ring[seen % kTileRing] : -1;
        ring_end = tl < 0;
        v = tl < 0 ? -1 : tl * kKeyTile;
      }
      ++seen;
      return v;
    };
    auto scales_of = [&](int base, float& ks, float& vs, bool& ok_row) {
      const long long row = base >= 0 ? entry_row(base + t) : -1;
      ok_row = row >= 0;
      ks = ok_row ? __ldg(p.kv.k_scale + row) : 0.f;
      vs = ok_row ? __ldg(p.kv.v_scale + row) : 0.f;
    };
    int base_next = next_base();
    int base_far = base_next >= 0 ? next_base() : -1;
    float ks_next, vs_next, ks_far, vs_far;
    bool val_next, val_far;
    scales_of(base_next, ks_next, vs_next, val_next);
    scales_of(base_far, ks_far, vs_far, val_far);
    const float qinv = qsc_s[0];
    const float c2 = p.sm_scale * kLog2eF8 * qinv;  // Q-scaled logit -> log2 units
    int n_done = 0;
    for (int i = 0;; ++i) {
      const int sb = i & 1;
      // This tile, and the one two ahead (its scales' loads start now).
      const int base = base_next;
      base_next = base_far;
      base_far = base_far >= 0 ? next_base() : -1;
      if (named_bar_or(3, NSOFT, !ok)) ok = false;
      if (!ok || base < 0) break;  // the same for every softmax thread
      n_done = i + 1;
      const int j = base + t;
      const float ks = ks_next, vs = vs_next;
      const bool valid = val_next;
      ks_next = ks_far;
      vs_next = vs_far;
      val_next = val_far;
      scales_of(base_far, ks_far, vs_far, val_far);
      if (ok && !mbar_wait(s_full + sb, (i >> 1) & 1)) ok = false;
      if (named_bar_or(3, NSOFT, !ok)) ok = false;
      tc_fence_after();
      float x[HH];
      {
        // Every chunk's load in flight before the one wait: the Q_hi columns, then Q_lo.
        uint32_t r[2 * HH];
#pragma unroll
        for (int c = 0; c < HH; c += 16) {
          tmem_ld16(tmem_base + lane_base + sb * 2 * H + hoff + c,
                    *reinterpret_cast<uint32_t(*)[16]>(r + c));
          tmem_ld16(tmem_base + lane_base + sb * 2 * H + H + hoff + c,
                    *reinterpret_cast<uint32_t(*)[16]>(r + HH + c));
        }
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < HH; ++e)
          x[e] = fmaf(__uint_as_float(r[HH + e]), 0.0625f, __uint_as_float(r[e]));
      }
      tc_fence_before();
      mbar_arrive(s_free + sb);
      if (!GATHER && p.sbuf) {
        if (j < k_end && j <= pos - p.window && pos - p.window + 1 > p.k_sel) {
          const float qk = qinv * ks;  // the stored logit is q.k times the key's scale
          float* dst = p.sbuf + ((size_t)bq * p.kv.max_len + j) * H + hoff;
#pragma unroll
          for (int e = 0; e < HH / 4; ++e) {
            uint4 v;
            v.x = __float_as_uint(x[4 * e] * qk);
            v.y = __float_as_uint(x[4 * e + 1] * qk);
            v.z = __float_as_uint(x[4 * e + 2] * qk);
            v.w = __float_as_uint(x[4 * e + 3] * qk);
            st_global_v4_hint(dst + 4 * e, v, keep_policy);
          }
        }
      }
      const float cks = c2 * ks;  // one Q scale for every head: one multiplier per key
#pragma unroll
      for (int e = 0; e < HH; ++e) x[e] = valid ? x[e] * cks : -INFINITY;
      if (sel_keys) {
        float u = x[0];
#pragma unroll
        for (int e = 1; e < HH; ++e) u = fmaxf(u, x[e]);
        const bool rec = valid && j < n_c;
        if (NHALF == 1) {
          if (rec) record_u(j, u);
        } else if (half == 1) {
          ux_s[(i & 1) * 128 + t] = u;
        } else {
          if (rec_prev) record_u(j_prev, fmaxf(u_prev, ux_s[((i - 1) & 1) * 128 + t]));
          u_prev = u;
          j_prev = j;
          rec_prev = rec;
        }
      }
      bool over = valid && fabsf(vs) > vlim;
#pragma unroll
      for (int h = 0; h < HH; ++h) over |= x[h] - ref(h) > kRescaleAtF8;
      if (group_bar_or(half, over)) {
        // Move the references to the tile maxima where these are higher, and the V
        // exponent to cover the largest |v_scale| of the tile; rescale l and O.
        {
          const float vm = warp_max(valid ? fabsf(vs) : 0.f);
          if (lane_id() == 0) red[4 * H + 4 * half + (t >> 5)] = vm;
        }
        block_max_group_f8<HH, H>(x, red, alpha_s, t, hoff, half);
        if (t < HH) {
          const int h = hoff + t;
          const float mnew = fmaxf(mref_s[h], alpha_s[h]);
          alpha_s[h] = exp2f(mref_s[h] - mnew);
          mref_s[h] = mnew;
        }
        if (t == 0) {
          const float* vr = red + 4 * H + 4 * half;
          const float vmax = fmaxf(fmaxf(vr[0], vr[1]), fmaxf(vr[2], vr[3]));
          const int e_old = ev_s[half];
          int e_new = e_old;
          if (vmax > 0.f) {
            int ex;
            frexpf(vmax, &ex);  // vmax < 2^ex
            ex = ex < -126 ? -126 : ex;
            if (ex > e_old) e_new = ex;
          }
          beta_s[half] = e_new == e_old ? 1.f : (e_old == kNoScale ? 0.f : ldexpf(1.f, e_old - e_new));
          ev_s[half] = e_new;
        }
        group_bar_sync(half);
        const float beta = beta_s[half];
        ev = ev_s[half];
        vlim = ev == kNoScale ? 0.f : ldexpf(1.f, ev);
        vmul = ev == kNoScale ? 0.f : ldexpf(1.f, -ev);
#pragma unroll
        for (int h = 0; h < HH; ++h) {
          l[h] *= alpha_s[hoff + h];
          if (kRefRegs) mr[kRefRegs ? h : 0] = mref_s[hoff + h];
        }
        if (i > 0) {
          if (ok && !mbar_wait(p_free + ((i - 1) & 1), ((i - 1) >> 1) & 1)) ok = false;
          tc_fence_after();
#pragma unroll
          for (int term = 0; term < 3; ++term) {
#pragma unroll
            for (int c = 0; c < HH; c += 16) {
              uint32_t r[16];
              tmem_ld16(tmem_o + lane_base + term * H + hoff + c, r);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 16; ++e)
                r[e] = __float_as_uint(__uint_as_float(r[e]) * (alpha_s[hoff + c + e] * beta));
              tmem_st16(tmem_o + lane_base + term * H + hoff + c, r);
            }
          }
          tmem_wait_st();
          tc_fence_before();
        }
      }
      if (ok && i >= 2 && !mbar_wait(p_free + sb, ((i >> 1) & 1) ^ 1)) ok = false;
      uint8_t* pb = ps + sb * L::kPBytes;
      const float vsc = valid ? vs * vmul : 0.f;
#pragma unroll
      for (int c = 0; c < HH / 16; ++c) {
        uint32_t w0[4], w1[4], w2[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          w0[e] = 0u;
          w1[e] = 0u;
          w2[e] = 0u;
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int h0 = c * 16 + 4 * e + 2 * u;
            // A head whose reference is still -inf has seen no key: its p is 0 (not
            // 2^(-inf - -inf)), so a leading all-padding tile leaves O and l at zero.
            const float p0 = ex2_ftz(x[h0] - finite_ref(ref(h0)));
            const float p1 = ex2_ftz(x[h0 + 1] - finite_ref(ref(h0 + 1)));
            l[h0] += p0;
            l[h0 + 1] += p1;
            uint32_t ch, cl, cl2;
            e4m3_split3(__floats2half2_rn(p0 * vsc, p1 * vsc), ch, cl, cl2);
            w0[e] |= ch << (16 * u);
            w1[e] |= cl << (16 * u);
            w2[e] |= cl2 << (16 * u);
          }
        }
        const int ch0 = (hoff >> 4) + c;  // chunk of this head group's 16 heads, term 0
        *reinterpret_cast<uint4*>(pb + ch0 * (kKeyTile * 16) + t * 16) =
            make_uint4(w0[0], w0[1], w0[2], w0[3]);
        *reinterpret_cast<uint4*>(pb + (ch0 + H / 16) * (kKeyTile * 16) + t * 16) =
            make_uint4(w1[0], w1[1], w1[2], w1[3]);
        *reinterpret_cast<uint4*>(pb + (ch0 + 2 * (H / 16)) * (kKeyTile * 16) + t * 16) =
            make_uint4(w2[0], w2[1], w2[2], w2[3]);
      }
      if (!GATHER && !valid && half == 0) {
        // Rows past the row's end (only its last tile has them) may hold anything, NaN
        // codes included; 0 * NaN would poison P.V, so zero this key's V row once its
        // tile has landed.
        const int s = i % R;
        if (ok && !mbar_wait(vr_full + s, (i / R) & 1)) ok = false;
        uint4* v0 = reinterpret_cast<uint4*>(vraw + s * kRawTile + t * 128);
#pragma unroll
        for (int e = 0; e < 8; ++e) v0[e] = make_uint4(0, 0, 0, 0);
      }
      fence_proxy_async_smem();
      mbar_arrive(p_full + sb);
    }
    if (NHALF == 2 && sel_keys) {
      named_bar_sync(3, NSOFT);
      if (half == 0 && rec_prev)
        record_u(j_prev, fmaxf(u_prev, ux_s[((n_done - 1) & 1) * 128 + t]));
    }
    // The merge kernel may be scheduled (it waits for this grid); with the fused tail the
    // next kernel starts only once the index set is written.
    if (GATHER || !p.fuse) griddep_launch_dependents();
    const int last = n_done - 1;
    if (ok && n_done > 0 && !mbar_wait(p_free + (last & 1), (last >> 1) & 1)) ok = false;
    tc_fence_after();
    const float oscale = ev == kNoScale ? 0.f : ldexpf(1.f, ev);
#pragma unroll
    for (int c = 0; c < HH; c += 16) {
      uint32_t r0[16], r1[16], r2[16];
      tmem_ld16(tmem_o + lane_base + hoff + c, r0);
      tmem_ld16(tmem_o + lane_base + H + hoff + c, r1);
      tmem_ld16(tmem_o + lane_base + 2 * H + hoff + c, r2);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float o = fmaf(__uint_as_float(r2[e]), 0.00390625f,
                             fmaf(__uint_as_float(r1[e]), 0.0625f, __uint_as_float(r0[e])));
        part_o[(hoff + c + e) * kHeadDim + t] = o * oscale;
      }
    }
    tc_fence_before();
#pragma unroll
    for (int h = 0; h < HH; ++h) {
      const float s = warp_sum(l[h]);
      if (lane_id() == 0) red[(warp & 3) * H + hoff + h] = s;
    }
    group_bar_sync(half);
    if (t < HH) {
      const int h = hoff + t;
      part_ml[2 * h] = mref_s[h];
      part_ml[2 * h + 1] = red[h] + red[H + h] + red[2 * H + h] + red[3 * H + h];
    }
  }
  }
  if (!ok) set_status(p.status, HS2_ERR_DEVICE_TIMEOUT);
  if (on_chip) {
    // Every CTA of the cluster reaches both barriers (no early exit above); the second
    // keeps each CTA's shared memory alive until the others have read it.
    __syncwarp();
    cluster_sync();
    griddep_wait();  // the previous grid is done before this layer writes its output
    cluster_merge_row<H>(smem, p.splits1, p.out + (size_t)bq * H * kHeadDim);
    __syncwarp();
    cluster_sync();
  }
  if constexpr (!GATHER) {
    if (p.fuse && !full_fp8_tail<H>(p)) set_status(p.status, HS2_ERR_DEVICE_TIMEOUT);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(*tmem_slot, L::kTmemCols);
  }
}

template <int H, bool GATHER>
static cudaError_t launch_fp8_t(FullParams p, const CUtensorMap& tk, const CUtensorMap& tv,
                                int bq, cudaStream_t st) {
  using L = Fp8Smem<H, GATHER>;
  auto kernel = full_attn_fp8_kernel<H, GATHER>;
  static int max_cluster = 0;
  if (!max_cluster) {
    cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
    if (e != cudaSuccess) return e;
    max_cluster = GATHER ? largest_cluster(kernel, dim3(fp8_threads<H>()), L::kBytes) : 1;
    if (max_cluster < 1) return cudaErrorLaunchOutOfResources;
  }
  if (!GATHER)
    return launch_pdl_coop(kernel, dim3(p.splits1, bq), dim3(fp8_threads<H>()), L::kBytes,
                           p.fuse != 0 && p.splits1 > 1, st, tk, tv, p);
  plan_gather_cluster(p.idx_width, max_cluster, &p.splits1, &p.chunk1);
  return launch_pdl_cluster(kernel, dim3(p.splits1, bq), dim3(fp8_threads<H>()), L::kBytes, p.splits1,
                            st, tk, tv, p);
}

template <bool GATHER>
static cudaError_t launch_fp8_h(const FullParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                                int bq, cudaStream_t st) {
  switch (p.h) {
    case 16: return launch_fp8_t<16, GATHER>(p, tk, tv, bq, st);
    case 32: return launch_fp8_t<32, GATHER>(p, tk, tv, bq, st);
    case 48: return launch_fp8_t<48, GATHER>(p, tk, tv, bq, st);
    case 64: return launch_fp8_t<64, GATHER>(p, tk, tv, bq, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_full_attn_fp8(const FullParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                                 int bq, cudaStream_t st) {
  return launch_fp8_h<false>(p, tk, tv, bq, st);
}

cudaError_t launch_sparse_attn_fp8(FullParams p, int bq, cudaStream_t st) {
  CUtensorMap unused;
  memset(&unused, 0, sizeof(unused));
  return launch_fp8_h<true>(p, unused, unused, bq, st);
}

}  // namespace hs2
