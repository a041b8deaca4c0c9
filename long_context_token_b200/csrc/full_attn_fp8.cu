// Full-attention layer (and, in gather mode, a reusing sparse layer) on the
// 5th-generation tensor cores for an FP8 E4M3 KV cache with per-token scales
// (web coverage of HySparse2: the 1M-token footprint is quoted with an FP8 KV cache;
// "Luo Fuli Teases Xiaomi MiMo-V3 Architecture ...", paragraph on cost at 1M tokens).
//
// The MMA needs both operands in the same 16-bit type.  E4M3 values are exact in f16
// (4 significant bits, exponents 2^-9 .. 2^8), so the codes are widened to f16 with no
// rounding; the per-token scales stay out of the MMA: k_scale[j] multiplies key j's
// logits and v_scale[j] multiplies its probability before P.V.  Q (bf16) becomes f16
// after a per-head power-of-two scaling that puts its largest element in [2^14, 2^15),
// so the conversion cannot overflow; the scale is divided out of the logits.
//
// One CTA per key chunk (or per 128 index entries) of one (sequence, token):
//   warp 0      producer: TMA of 128-row E4M3 tiles (128-byte rows, 128-byte
//               swizzle) into an R-stage raw ring; in gather mode cp.async of the
//               indexed rows into the same layout;
//   warp 1      TMEM allocator and MMA issuer (kind::f16 with f16 inputs):
//                 S^T[128 keys x H] = K16 . Q16^T,   O^T[128 d x H] += V16^T . P16^T;
//   warps 2..5  softmax, as in the bf16 kernel (one key per thread, lazily moved
//               per-head reference), P in f16;
//   warps 6..9  conversion: raw K / V tiles -> f16 in the swizzled operand layout
//               (rows past the chunk end or absent in the index are zeroed).
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <string.h>

#include "hs2_internal.cuh"
#include "sm100.cuh"
#include "tc_common.cuh"

namespace hs2 {

using namespace sm100;

namespace {

constexpr float kLog2eF8 = 1.4426950408889634f;
constexpr float kRescaleAtF8 = 8.0f;
// Conversion warps: eight (four for K rows, four for V rows, converting in parallel on
// their own barriers) up to 32 heads; four (each thread a K row, then a V row) above,
// where the softmax registers leave no room for more threads.
template <int H>
__host__ __device__ constexpr int fp8_conv_warps() { return H <= 32 ? 8 : 4; }
// Softmax threads per key: two at 64 heads (each takes 32 of the key's heads, so that
// its logits and running sums stay in registers), else one.
template <int H>
__host__ __device__ constexpr int fp8_halves() { return H == 64 ? 2 : 1; }
template <int H>
__host__ __device__ constexpr int fp8_threads() {
  return 64 + 128 * fp8_halves<H>() + 32 * fp8_conv_warps<H>();
}
constexpr uint32_t kRawTile = 16384;    // 128 keys x 128 E4M3 codes
constexpr uint32_t kConvTile = 32768;   // 128 keys x 128 f16 (two 64-column boxes)

// Gather mode (a sparse layer) keeps one raw stage and one converted V buffer: its CTAs
// mostly take a single tile, and the smaller footprint lets two CTAs share an SM.
template <int H, bool GATHER>
struct Fp8Smem {
  static constexpr int R = GATHER ? 1 : (H <= 16 ? 3 : 2);  // raw stages (K and V each)
  static constexpr int kVConv = GATHER ? 1 : 2;              // converted V buffers
  static constexpr uint32_t kQBytes = H * kHeadDim * 2;
  static constexpr uint32_t kPBytes = kKeyTile * H * 2;
  static constexpr uint32_t kKRawOff = 0;
  static constexpr uint32_t kVRawOff = R * kRawTile;
  static constexpr uint32_t kKConvOff = 2 * R * kRawTile;
  static constexpr uint32_t kVConvOff = kKConvOff + kConvTile;
  static constexpr uint32_t kQOff = kVConvOff + kVConv * kConvTile;
  static constexpr uint32_t kPOff = kQOff + kQBytes;          // [2 buffers]
  static constexpr uint32_t kRedOff = kPOff + 2 * kPBytes;    // [4 warps][H]
  static constexpr uint32_t kRefOff = kRedOff + 4 * H * 4;    // mref, alpha, c2, qinv
  static constexpr uint32_t kBarOff = kRefOff + 4 * H * 4;
  static constexpr uint32_t kBars = 4 * R + 15;
  static constexpr uint32_t kSlotOff = kBarOff + kBars * 8;
  static constexpr uint32_t kBytes = kSlotOff + 16 + 1024;
  static constexpr uint32_t kTmemCols = tmem_cols_pow2(3 * H);
  static_assert(kBytes <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_codes) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)two_codes, __NV_E4M3);
  return (uint32_t)h.x | ((uint32_t)h.y << 16);
}

// Raw tile (128 rows x 128 codes, 16-byte chunk c of row r at chunk c ^ (r & 7)) ->
// f16 tile in two 64-column boxes with the same swizzle.  Thread t (0..127) converts
// row t; rows with valid == false become zeros.
__device__ __forceinline__ void convert_row(const uint8_t* raw, uint8_t* conv, int r, bool valid) {
  const uint8_t* src = raw + r * 128;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint4 in = *reinterpret_cast<const uint4*>(src + (((c ^ r) & 7) << 4));
    uint32_t w[4] = {in.x, in.y, in.z, in.w};
    uint32_t o[8];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      o[2 * u] = valid ? e4m3x2_to_f16x2(w[u] & 0xffffu) : 0u;
      o[2 * u + 1] = valid ? e4m3x2_to_f16x2(w[u] >> 16) : 0u;
    }
    // f16 elements 16c .. 16c+15: box c >> 2, 16-byte chunks 2(c & 3) and 2(c & 3) + 1.
    uint8_t* dst = conv + (c >> 2) * kBoxBytes + r * 128;
    const int c0 = 2 * (c & 3);
    *reinterpret_cast<uint4*>(dst + (((c0 ^ r) & 7) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
    *reinterpret_cast<uint4*>(dst + ((((c0 + 1) ^ r) & 7) << 4)) =
        make_uint4(o[4], o[5], o[6], o[7]);
  }
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

template <int H>
__device__ __forceinline__ void block_max_heads_f8(const float (&v)[H], float* red, float* out,
                                                   int t) {
  const int w = t >> 5, lane = t & 31;
#pragma unroll
  for (int h = 0; h < H; ++h) {
    const float m = warp_max(v[h]);
    if (lane == 0) red[w * H + h] = m;
  }
  named_bar_sync(1, 128);
  if (t < H) out[t] = fmaxf(fmaxf(red[t], red[H + t]), fmaxf(red[2 * H + t], red[3 * H + t]));
  named_bar_sync(1, 128);
}

}  // namespace

template <int H, bool GATHER>
__global__ void __launch_bounds__(fp8_threads<H>(), 1)
    full_attn_fp8_kernel(const __grid_constant__ CUtensorMap tmap_k,
                         const __grid_constant__ CUtensorMap tmap_v, FullParams p) {
  using L = Fp8Smem<H, GATHER>;
  constexpr int R = L::R;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* kraw = smem + L::kKRawOff;
  uint8_t* vraw = smem + L::kVRawOff;
  uint8_t* kconv = smem + L::kKConvOff;
  uint8_t* vconv = smem + L::kVConvOff;
  uint8_t* qs = smem + L::kQOff;
  uint8_t* ps = smem + L::kPOff;
  float* red = reinterpret_cast<float*>(smem + L::kRedOff);
  float* mref_s = reinterpret_cast<float*>(smem + L::kRefOff);
  float* alpha_s = mref_s + H;
  float* c2_s = mref_s + 2 * H;    // sm_scale * log2(e) / (Q scale of head h)
  float* qinv_s = mref_s + 3 * H;  // 1 / (Q scale of head h)
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* kr_full = bars;
  uint64_t* kr_empty = bars + R;
  uint64_t* vr_full = bars + 2 * R;
  uint64_t* vr_empty = bars + 3 * R;
  uint64_t* kc_full = bars + 4 * R;      // [1]
  uint64_t* kc_empty = kc_full + 1;      // [1]
  uint64_t* vc_full = kc_full + 2;       // [2]
  uint64_t* vc_empty = kc_full + 4;      // [2]
  uint64_t* s_full = kc_full + 6;        // [2]
  uint64_t* s_free = kc_full + 8;        // [2]
  uint64_t* p_full = kc_full + 10;       // [2]
  uint64_t* p_free = kc_full + 12;       // [2]
  uint64_t* mma_done = kc_full + 14;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kSlotOff);

  const int warp = threadIdx.x >> 5;
  const int split = blockIdx.x, bq = blockIdx.y;
  const int b = bq / p.n_q, qi = bq % p.n_q;

  // Set-up that touches no global memory, overlapping the previous kernel's tail.
  if (threadIdx.x == 0) {
    for (int s = 0; s < R; ++s) {
      mbar_init(kr_full + s, GATHER ? 32 : 1);
      mbar_init(kr_empty + s, 128);
      mbar_init(vr_full + s, GATHER ? 32 : 1);
      mbar_init(vr_empty + s, 128);
    }
    mbar_init(kc_full, 128);
    mbar_init(kc_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(vc_full + s, 128);
      mbar_init(vc_empty + s, 1);
      mbar_init(s_full + s, 1);
      mbar_init(s_free + s, 128 * fp8_halves<H>());
      mbar_init(p_full + s, 128 * fp8_halves<H>());
      mbar_init(p_free + s, 1);
    }
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
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
  const int n_tiles = k0 < k1 ? (k1 - k0 + kKeyTile - 1) / kKeyTile : 0;
  const size_t pidx = (size_t)bq * p.splits1 + split;

  // Row of the cache behind tile entry e (or -1 for an absent / past-the-end entry).
  auto entry_row = [&](int e) -> long long {
    if (e >= k1) return -1;
    if (!GATHER) return (long long)(row_base + e);
    const int j = __ldcg(idx_row + e);  // through L2: may have been written by the previous grid
    return (j >= 0 && j < Lb) ? (long long)(row_base + j) : -1;
  };
  bool ok = true;
  // Cluster mode keeps the partial in this CTA's shared memory (the raw stages, idle by
  // the time the partial is written) for the on-chip merge.
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
    // The first tile's rows are gathered by every thread of the CTA; warp 0 gathers any
    // later tiles.  (store_q_f16_scaled below synchronises the block.)
    gather_tile_rows<8, kRawTile>(smem_u32(kraw), smem_u32(vraw),
                                  static_cast<const uint8_t*>(p.kv.k),
                                  static_cast<const uint8_t*>(p.kv.v), idx_row, k0, k1, Lb,
                                  row_base, p.status, threadIdx.x, blockDim.x);
  }
  // Q in f16 under a per-head power-of-two scale; its inverse goes into the logits.
  store_q_f16_scaled<H>(qs, p.q + (size_t)bq * H * kHeadDim, qinv_s, nullptr);
  if (GATHER) cp_async_wait_all();
  for (int h = threadIdx.x; h < H; h += blockDim.x) c2_s[h] = p.sm_scale * kLog2eF8 * qinv_s[h];
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t tmem_o = tmem_base + 2 * H;

  if (warp == 0) {
    if (GATHER) {
      // ---------------------------------------------- gather producer (32 lanes)
      const int lane = (int)lane_id();
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i % R;
        if (i > 0) {  // tile 0 was gathered by the whole CTA above
          const uint32_t ph = ((i / R) & 1) ^ 1;
          if (ok && !mbar_wait(kr_empty + s, ph)) ok = false;
          if (ok && !mbar_wait(vr_empty + s, ph)) ok = false;
          gather_tile_rows<8, kRawTile>(
              smem_u32(kraw + s * kRawTile), smem_u32(vraw + s * kRawTile),
              static_cast<const uint8_t*>(p.kv.k), static_cast<const uint8_t*>(p.kv.v), idx_row,
              k0 + i * kKeyTile, k1, Lb, row_base, p.status, lane, 32);
          cp_async_wait_all();
          fence_proxy_async_smem();
        }
        mbar_arrive(kr_full + s);
        mbar_arrive(vr_full + s);
      }
    } else if (elect_one()) {
      // ---------------------------------------------------------- TMA producer
      const uint64_t pol = policy_evict_first();
      const int row0 = b * p.kv.max_len + k0;
      int issued = 0;
      for (int i = 0; i < n_tiles && ok; ++i) {
        const int s = i % R;
        const uint32_t ph = ((i / R) & 1) ^ 1;
        const int row = row0 + i * kKeyTile;
        if (!mbar_wait(kr_empty + s, ph)) { ok = false; break; }
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
      const uint32_t id_qk = idesc_f16(128, H, false, false, false);
      const uint32_t id_pv = idesc_f16(128, H, false, true, true);
      const uint32_t q_addr = smem_u32(qs);
      const uint32_t k_addr = smem_u32(kconv);
      auto issue_pv = [&](int t) -> bool {
        const int vb = t % L::kVConv, pb = t & 1;
        if (!mbar_wait(vc_full + vb, (t / L::kVConv) & 1)) return false;
        if (!mbar_wait(p_full + pb, (t >> 1) & 1)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(vconv + vb * kConvTile);
        const uint32_t p_addr = smem_u32(ps + pb * L::kPBytes);
#pragma unroll
        for (int kk = 0; kk < kKeyTile / 16; ++kk)
          mma_f16_ss(tmem_o, vt_mnmajor_sw128_desc(v_addr, kk), pt_mnmajor_desc(p_addr, kk),
                     id_pv, (t > 0 || kk > 0) ? 1u : 0u);
        mma_commit(p_free + pb);
        mma_commit(vc_empty + vb);
        return true;
      };
      for (int i = 0; i < n_tiles && ok; ++i) {
        const int sb = i & 1;
        if (!mbar_wait(kc_full, i & 1)) { ok = false; break; }
        if (!mbar_wait(s_free + sb, ((i >> 1) & 1) ^ 1)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kHeadDim / 16; ++kk)
          mma_f16_ss(tmem_base + sb * H, kmajor_sw128_desc(k_addr, kk),
                     q_kmajor_desc<H>(q_addr, kk), id_qk, kk > 0 ? 1u : 0u);
        mma_commit(s_full + sb);
        mma_commit(kc_empty);
        if (i > 0 && !issue_pv(i - 1)) { ok = false; break; }
      }
      if (ok && !issue_pv(n_tiles - 1)) ok = false;
      mma_commit(mma_done);
      if (!mbar_wait(mma_done, 0)) ok = false;
    }
  } else if (warp >= 2 + 4 * fp8_halves<H>()) {
    // ------------------------------------------------------------ conversion
    const int ct = threadIdx.x - (64 + 128 * fp8_halves<H>());
    const int t = ct & (kKeyTile - 1);  // row of the tile
    constexpr bool kSplit = fp8_conv_warps<H>() == 8;
    const bool do_k = !kSplit || ct < kKeyTile, do_v = !kSplit || ct >= kKeyTile;
    for (int i = 0; i < n_tiles; ++i) {
      const int s = i % R;
      const bool valid = entry_row(k0 + i * kKeyTile + t) >= 0;
      if (do_k) {
        if (ok && !mbar_wait(kr_full + s, (i / R) & 1)) ok = false;
        if (ok && !mbar_wait(kc_empty, (i & 1) ^ 1)) ok = false;
        convert_row(kraw + s * kRawTile, kconv, t, valid);
        fence_proxy_async_smem();
        mbar_arrive(kc_full);
        mbar_arrive(kr_empty + s);
      }
      if (do_v) {
        const int vb = i % L::kVConv;
        if (ok && !mbar_wait(vr_full + s, (i / R) & 1)) ok = false;
        if (ok && !mbar_wait(vc_empty + vb, ((i / L::kVConv) & 1) ^ 1)) ok = false;
        convert_row(vraw + s * kRawTile, vconv + vb * kConvTile, t, valid);
        fence_proxy_async_smem();
        mbar_arrive(vc_full + vb);
        mbar_arrive(vr_empty + s);
      }
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
    float l[HH];
#pragma unroll
    for (int h = 0; h < HH; ++h) l[h] = 0.f;
    if (t < HH) mref_s[hoff + t] = -INFINITY;
    group_bar_sync(half);
    // Per-key scales (and validity) are loaded two tiles ahead so that their memory
    // latency overlaps the tiles in between instead of stalling each tile.
    auto scales_of = [&](int i, float& ks, float& vs, bool& ok_row) {
      const long long row = i < n_tiles ? entry_row(k0 + i * kKeyTile + t) : -1;
      ok_row = row >= 0;
      ks = ok_row ? __ldg(p.kv.k_scale + row) : 0.f;
      vs = ok_row ? __ldg(p.kv.v_scale + row) : 0.f;
    };
    float ks_next, vs_next, ks_far, vs_far;
    bool val_next, val_far;
    scales_of(0, ks_next, vs_next, val_next);
    scales_of(1, ks_far, vs_far, val_far);
    const float c2 = c2_s[0];  // sm_scale * log2(e) / (the Q scale, common to all heads)
    for (int i = 0; i < n_tiles; ++i) {
      const int sb = i & 1;
      const int j = k0 + i * kKeyTile + t;
      const float ks = ks_next, vs = vs_next;
      const bool valid = val_next;
      ks_next = ks_far;
      vs_next = vs_far;
      val_next = val_far;
      scales_of(i + 2, ks_far, vs_far, val_far);
      if (ok && !mbar_wait(s_full + sb, (i >> 1) & 1)) ok = false;
      if (named_bar_or(3, NSOFT, !ok)) ok = false;
      tc_fence_after();
      float x[HH];
      {
        // Every chunk's load in flight before the one wait.
        uint32_t r[HH];
#pragma unroll
        for (int c = 0; c < HH; c += 16)
          tmem_ld16(tmem_base + lane_base + sb * H + hoff + c,
                    *reinterpret_cast<uint32_t(*)[16]>(r + c));
        tmem_wait_ld();
        if (!GATHER && p.sbuf) {
          if (j < k1 && j <= pos - p.window && pos - p.window + 1 > p.k_sel) {
            float* dst = p.sbuf + ((size_t)bq * p.kv.max_len + j) * H + hoff;
#pragma unroll
            for (int e = 0; e < HH / 4; ++e) {
              uint4 v;
              v.x = __float_as_uint(__uint_as_float(r[4 * e]) * qinv_s[hoff + 4 * e] * ks);
              v.y = __float_as_uint(__uint_as_float(r[4 * e + 1]) * qinv_s[hoff + 4 * e + 1] * ks);
              v.z = __float_as_uint(__uint_as_float(r[4 * e + 2]) * qinv_s[hoff + 4 * e + 2] * ks);
              v.w = __float_as_uint(__uint_as_float(r[4 * e + 3]) * qinv_s[hoff + 4 * e + 3] * ks);
              st_global_v4_hint(dst + 4 * e, v, keep_policy);
            }
          }
        }
        const float cks = c2 * ks;  // one Q scale for every head: one multiplier per key
#pragma unroll
        for (int e = 0; e < HH; ++e) x[e] = valid ? __uint_as_float(r[e]) * cks : -INFINITY;
      }
      tc_fence_before();
      mbar_arrive(s_free + sb);
      // This group's references: read once per tile into registers up to 16 heads per
      // thread; above, from shared memory at each use (registers are the limit there).
      constexpr bool kRefRegs = HH <= 16;
      float mr[kRefRegs ? HH : 1];
      if (kRefRegs) {
#pragma unroll
        for (int h = 0; h < HH; ++h) mr[h] = mref_s[hoff + h];
      }
      auto ref = [&](int h) { return kRefRegs ? mr[kRefRegs ? h : 0] : mref_s[hoff + h]; };
      bool over = false;
#pragma unroll
      for (int h = 0; h < HH; ++h) over |= x[h] - ref(h) > kRescaleAtF8;
      if (group_bar_or(half, over)) {
        block_max_group_f8<HH, H>(x, red, alpha_s, t, hoff, half);
        if (t < HH) {
          const int h = hoff + t;
          const float mnew = fmaxf(mref_s[h], alpha_s[h]);
          alpha_s[h] = exp2f(mref_s[h] - mnew);
          mref_s[h] = mnew;
        }
        group_bar_sync(half);
#pragma unroll
        for (int h = 0; h < HH; ++h) {
          l[h] *= alpha_s[hoff + h];
          if (kRefRegs) mr[kRefRegs ? h : 0] = mref_s[hoff + h];
        }
        if (i > 0) {
          if (ok && !mbar_wait(p_free + ((i - 1) & 1), ((i - 1) >> 1) & 1)) ok = false;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < HH; c += 16) {
            uint32_t r[16];
            tmem_ld16(tmem_o + lane_base + hoff + c, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e)
              r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha_s[hoff + c + e]);
            tmem_st16(tmem_o + lane_base + hoff + c, r);
          }
          tmem_wait_st();
          tc_fence_before();
        }
      }
      if (ok && i >= 2 && !mbar_wait(p_free + sb, ((i >> 1) & 1) ^ 1)) ok = false;
      uint8_t* pb = ps + sb * L::kPBytes;
#pragma unroll
      for (int c = 0; c < HH / 8; ++c) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int h0 = c * 8 + 2 * e;
          // A head whose reference is still -inf has seen no key: its p is 0 (not
          // 2^(-inf - -inf)), so a leading all-padding tile leaves O and l at zero.
          const float p0 = ex2_ftz(x[h0] - finite_ref(ref(h0)));
          const float p1 = ex2_ftz(x[h0 + 1] - finite_ref(ref(h0 + 1)));
          l[h0] += p0;
          l[h0 + 1] += p1;
          const __half2 v2 = __floats2half2_rn(p0 * vs, p1 * vs);
          w[e] = *reinterpret_cast<const uint32_t*>(&v2);
        }
        *reinterpret_cast<uint4*>(pb + (hoff / 8 + c) * (kKeyTile * 16) + t * 16) =
            make_uint4(w[0], w[1], w[2], w[3]);
      }
      fence_proxy_async_smem();
      mbar_arrive(p_full + sb);
    }
    griddep_launch_dependents();  // the merge may be scheduled; it waits for this grid
    const int last = n_tiles - 1;
    if (ok && !mbar_wait(p_free + (last & 1), (last >> 1) & 1)) ok = false;
    tc_fence_after();
#pragma unroll
    for (int c = 0; c < HH; c += 16) {
      uint32_t r[16];
      tmem_ld16(tmem_o + lane_base + hoff + c, r);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 16; ++e)
        part_o[(hoff + c + e) * kHeadDim + t] = __uint_as_float(r[e]);
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
    return launch_pdl(kernel, dim3(p.splits1, bq), dim3(fp8_threads<H>()), L::kBytes, st, tk, tv,
                      p);
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
