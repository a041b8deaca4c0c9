// Importance pass on the 5th-generation tensor cores (bf16 cache).
//
// Selection keys t_j = max_h (s_hj - delta_h) for the keys outside the window
// (importance of a key = its largest softmax probability over the query heads;
// the full layer's scores drive the token selection -- toolnavs article 2080, fr
// "Ce que fait HySparse2"), plus a 12-bit radix histogram of t's order-preserving
// key in shared memory, flushed to the per-query global histogram.
//
// One CTA per key chunk of one (sequence, query token).  Warp roles:
//   warp 0      TMA producer: 128-key K tiles (two 64-column boxes, 128-byte
//               swizzle) into an NS-stage ring;
//   warp 1      TMEM allocator and MMA issuer: S^T[128 keys x H] = K_tile . Q^T,
//               eight K=16 steps of tcgen05.mma kind::f16 into one of two TMEM
//               buffers;
//   warps 2..5  epilogue: thread t owns TMEM lane t (= key t of the tile), loads
//               its H logits, takes the max over heads, writes t_j and counts it.
#include "hs2_internal.cuh"
#include "sm100.cuh"
#include "tc_common.cuh"
#include "tile_simt.cuh"

namespace hs2 {

using namespace sm100;

template <int H>
struct ImpSmem {
  static constexpr int kStages = 4;
  static constexpr uint32_t kTileBytes = kKTileBytesBf16;  // 32 KB
  static constexpr uint32_t kQBytes = H * kHeadDim * 2;
  // offsets from a 1024-aligned base
  static constexpr uint32_t kStageOff = 0;
  static constexpr uint32_t kQOff = kStages * kTileBytes;
  static constexpr uint32_t kHistOff = kQOff + kQBytes;
  static constexpr uint32_t kDeltaOff = kHistOff + kHistBins * 4;
  static constexpr uint32_t kBarOff = kDeltaOff + H * 4;
  static constexpr uint32_t kBars = 2 * kStages + 5;
  static constexpr uint32_t kTmemSlotOff = kBarOff + kBars * 8;
  static constexpr uint32_t kBytes = kTmemSlotOff + 16 + 1024;  // + alignment slack
  static constexpr uint32_t kTmemCols = tmem_cols_pow2(2 * H);
};

template <int H>
__global__ void __launch_bounds__(192, 1)
    importance_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, SelectParams p) {
  using L = ImpSmem<H>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* stages = smem + L::kStageOff;
  uint8_t* qs = smem + L::kQOff;
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(smem + L::kHistOff);
  float* delta_s = reinterpret_cast<float*>(smem + L::kDeltaOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* full = bars;                  // [kStages]
  uint64_t* empty = bars + L::kStages;    // [kStages]
  uint64_t* s_full = bars + 2 * L::kStages;      // [2]
  uint64_t* s_free = bars + 2 * L::kStages + 2;  // [2]
  uint64_t* mma_done = bars + 2 * L::kStages + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlotOff);

  const int warp = threadIdx.x >> 5;
  const int split = blockIdx.x, bq = blockIdx.y;
  const int b = bq / p.n_q, qi = bq % p.n_q;
  const int Lb = seq_len(p.kv, b, p.n_q, p.status, false);
  const int pos = Lb - p.n_q + qi;
  const int n_c = pos - p.window + 1;
  if (n_c <= p.k_sel) return;  // every outside key is kept: nothing to rank
  const int k0 = split * p.chunk2;
  const int k1 = min(k0 + p.chunk2, n_c);
  if (k0 >= k1) return;
  const int n_tiles = (k1 - k0 + kKeyTile - 1) / kKeyTile;

  // ---- set-up: barriers, TMEM, Q (K-major, no swizzle), delta, histogram
  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(s_full + s, 1);
      mbar_init(s_free + s, 128);
    }
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane_id() == 0) prefetch_tmap(&tmap_k);
  store_q_kmajor<H>(qs, p.q + (size_t)bq * H * kHeadDim, threadIdx.x, blockDim.x);
  for (int e = threadIdx.x; e < kHistBins; e += blockDim.x) hist_s[e] = 0u;
  load_delta(p.lse64 + (size_t)bq * H, H, delta_s, nullptr);
  fence_proxy_async_smem();  // Q written by threads, read by the tensor cores
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  bool ok = true;

  if (warp == 0) {
    // ---------------- TMA producer
    if (elect_one()) {
      const uint64_t pol = policy_evict_first();
      const int row0 = b * p.kv.max_len + k0;
      int issued = 0;
      for (int i = 0; i < n_tiles && ok; ++i) {
        const int s = i % L::kStages;
        const uint32_t ph = (i / L::kStages) & 1;
        if (!mbar_wait(empty + s, ph ^ 1)) { ok = false; break; }
        mbar_arrive_expect_tx(full + s, L::kTileBytes);
        uint8_t* dst = stages + s * L::kTileBytes;
        tma_load_2d(dst, &tmap_k, full + s, 0, row0 + i * kKeyTile, pol);
        tma_load_2d(dst + kBoxBytes, &tmap_k, full + s, 64, row0 + i * kKeyTile, pol);
        issued = i + 1;
      }
      // Every copy into this CTA's shared memory has landed before the CTA can exit.
      for (int i = issued > L::kStages ? issued - L::kStages : 0; i < issued; ++i)
        if (!mbar_wait(full + (i % L::kStages), (i / L::kStages) & 1)) ok = false;
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (elect_one()) {
      const uint32_t idesc = idesc_f16(128, H, true, false, false);
      const uint32_t q_addr = smem_u32(qs);
      for (int i = 0; i < n_tiles && ok; ++i) {
        const int s = i % L::kStages;
        const uint32_t ph = (i / L::kStages) & 1;
        const int buf = i & 1;
        if (!mbar_wait(full + s, ph)) { ok = false; break; }
        if (!mbar_wait(s_free + buf, ((i >> 1) & 1) ^ 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(stages + s * L::kTileBytes);
        const uint32_t d_tmem = tmem_base + buf * H;
#pragma unroll
        for (int kk = 0; kk < kHeadDim / 16; ++kk) {
          const uint64_t a = kmajor_sw128_desc(a_addr, kk);
          const uint64_t bdesc = q_kmajor_desc<H>(q_addr, kk);
          mma_f16_ss(d_tmem, a, bdesc, idesc, kk > 0 ? 1u : 0u);
        }
        mma_commit(s_full + buf);
        mma_commit(empty + s);
      }
      // Every MMA has finished before TMEM is released.
      mma_commit(mma_done);
      if (!mbar_wait(mma_done, 0)) ok = false;
    }
  } else {
    // ---------------- epilogue: 128 threads, one key each
    const int lg = warp & 3;                 // TMEM lane group of this warp
    const int t = lg * 32 + (int)lane_id();  // key within the tile
    float* trow = p.tbuf + (size_t)bq * p.kv.max_len;
    const float sc = p.sm_scale;
    for (int i = 0; i < n_tiles; ++i) {
      const int buf = i & 1;
      // After a failed wait the loop keeps its shape (warp-wide ops stay converged)
      // but waits no more.
      if (ok && !mbar_wait(s_full + buf, (i >> 1) & 1)) ok = false;
      tc_fence_after();
      float best = -INFINITY;
      const uint32_t taddr = tmem_base + ((uint32_t)(lg * 32) << 16) + buf * H;
#pragma unroll
      for (int c = 0; c < H; c += 16) {
        uint32_t r[16];
        tmem_ld16(taddr + c, r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e)
          best = fmaxf(best, __uint_as_float(r[e]) * sc - delta_s[c + e]);
      }
      tc_fence_before();
      mbar_arrive(s_free + buf);
      const int j = k0 + i * kKeyTile + t;
      const bool valid = j < k1;
      if (valid) trow[j] = best;
      const uint32_t bin = valid ? (ordered_key(best) >> kHistShift) : 0xFFFFFFFFu;
      const unsigned grp = __match_any_sync(0xffffffffu, bin);
      if (valid && (int)lane_id() == __ffs(grp) - 1) atomicAdd(hist_s + bin, __popc(grp));
    }
    named_bar_sync(1, 128);
    uint32_t* gh = p.hist + (size_t)bq * kHistBins;
    for (int e = t; e < kHistBins; e += 128)
      if (hist_s[e]) atomicAdd(gh + e, hist_s[e]);
  }
  if (!ok) set_status(p.status, HS2_ERR_DEVICE_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

template <int H>
static cudaError_t launch_imp_t(const SelectParams& p, const CUtensorMap& tm, int bq,
                                cudaStream_t st) {
  using L = ImpSmem<H>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(importance_tc_kernel<H>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  importance_tc_kernel<H><<<dim3(p.splits2, bq), 192, L::kBytes, st>>>(tm, p);
  return cudaGetLastError();
}

cudaError_t launch_importance_tc(const SelectParams& p, const CUtensorMap& tmap_k, int bq,
                                 cudaStream_t st) {
  switch (p.h) {
    case 16: return launch_imp_t<16>(p, tmap_k, bq, st);
    case 32: return launch_imp_t<32>(p, tmap_k, bq, st);
    case 48: return launch_imp_t<48>(p, tmap_k, bq, st);
    case 64: return launch_imp_t<64>(p, tmap_k, bq, st);
    case 80: return launch_imp_t<80>(p, tmap_k, bq, st);
    case 96: return launch_imp_t<96>(p, tmap_k, bq, st);
    case 112: return launch_imp_t<112>(p, tmap_k, bq, st);
    case 128: return launch_imp_t<128>(p, tmap_k, bq, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace hs2
