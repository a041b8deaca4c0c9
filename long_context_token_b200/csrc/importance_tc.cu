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
#include <cuda_fp16.h>
#include <cuda_fp8.h>

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
  griddep_wait();
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
      for (int c0 = 0; c0 < H; c0 += 64) {  // up to four loads in flight per wait
        uint32_t r[64];
#pragma unroll
        for (int c = 0; c < 64; c += 16)
          if (c0 + c < H) tmem_ld16(taddr + c0 + c, *reinterpret_cast<uint32_t(*)[16]>(r + c));
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 64; ++e)
          if (c0 + e < H) best = fmaxf(best, __uint_as_float(r[e]) * sc - delta_s[c0 + e]);
      }
      tc_fence_before();
      mbar_arrive(s_free + buf);
      const int j = k0 + i * kKeyTile + t;
      const bool valid = j < k1;
      if (valid) trow[j] = best;
      if (valid) atomicAdd(hist_s + (ordered_key(best) >> kHistShift), 1u);
    }
    named_bar_sync(1, 128);
    __shared__ uint32_t flush_red[128 + 1];
    flush_hist_top<128>(hist_s, p.hist + (size_t)bq * kHistBins, p.k_sel, t, flush_red,
                        [] { named_bar_sync(1, 128); });
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
  return launch_pdl(importance_tc_kernel<H>, dim3(p.splits2, bq), dim3(192), L::kBytes, st, tm, p);
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


// ============================================================================
// Several new tokens of one sequence per CTA (bf16 cache, the several-token full
// layer's shapes): S^T[128 keys x N] = K_tile . Q^T with N = G tokens x H heads
// (G = 128 / H), so each K tile is read once for G tokens.  Thread t (key t) takes,
// per token, the max over that token's H heads; each token has its own histogram,
// kept in shared memory as two 16-bit counters per word (a CTA's chunk is below
// 65536 keys, so a counter cannot carry into its neighbour).
// ============================================================================
namespace {

constexpr int kImpMqRows = 128;
constexpr int kImpMqMaxChunk = 65535;

template <int H>
struct ImpMqSmem {
  static constexpr int G = kImpMqRows / H;
  static constexpr int N = G * H;                          // MMA N (query rows)
  static constexpr int kStages = 3;
  static constexpr uint32_t kTileBytes = kKTileBytesBf16;  // 32 KB
  static constexpr uint32_t kQBytes = N * kHeadDim * 2;
  static constexpr uint32_t kStageOff = 0;
  static constexpr uint32_t kQOff = kStages * kTileBytes;
  static constexpr uint32_t kHistOff = kQOff + kQBytes;     // [G][kHistBins / 2] words
  static constexpr uint32_t kDeltaOff = kHistOff + G * (kHistBins / 2) * 4;
  static constexpr uint32_t kBarOff = kDeltaOff + N * 4;
  static constexpr uint32_t kBars = 2 * kStages + 5;
  static constexpr uint32_t kTmemSlotOff = kBarOff + kBars * 8;
  static constexpr uint32_t kBytes = kTmemSlotOff + 16 + 1024;
  static constexpr uint32_t kTmemCols = tmem_cols_pow2(2 * N);
  static_assert(kBytes <= 227 * 1024, "shared memory budget");
};

}  // namespace

template <int H>
__global__ void __launch_bounds__(192, 1)
    importance_mq_kernel(const __grid_constant__ CUtensorMap tmap_k, SelectParams p,
                         int n_groups) {
  using L = ImpMqSmem<H>;
  constexpr int G = L::G, N = L::N;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* stages = smem + L::kStageOff;
  uint8_t* qs = smem + L::kQOff;
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(smem + L::kHistOff);
  float* delta_s = reinterpret_cast<float*>(smem + L::kDeltaOff);  // [G][H]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* full = bars;
  uint64_t* empty = bars + L::kStages;
  uint64_t* s_full = bars + 2 * L::kStages;
  uint64_t* s_free = bars + 2 * L::kStages + 2;
  uint64_t* mma_done = bars + 2 * L::kStages + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kTmemSlotOff);

  const int warp = threadIdx.x >> 5;
  const int split = blockIdx.x;
  const int grp = blockIdx.y % n_groups, b = blockIdx.y / n_groups;
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
  griddep_wait();

  const int t0 = grp * G;
  const int ntok = min(G, p.n_q - t0);
  const int Lb = seq_len(p.kv, b, p.n_q, p.status, false);
  // Token g ranks the keys [0, n_c(g)), n_c(g) = p_g - window + 1; the group's last
  // token has the longest range.  Tokens with n_c <= k_sel keep everything.
  const int nc0 = Lb - p.n_q + t0 - p.window + 1;  // n_c of token t0
  const int nc_last = nc0 + ntok - 1;
  const int k0 = split * p.chunk2;
  const int k1 = min(k0 + p.chunk2, nc_last);
  const bool any_ranked = nc_last > p.k_sel && k0 < k1;
  const int n_tiles = any_ranked ? (k1 - k0 + kKeyTile - 1) / kKeyTile : 0;

  if (n_tiles > 0) {
    // Q rows (token g, head h) at row g * H + h, K-major unswizzled; absent tokens zero.
    for (int e = threadIdx.x; e < N * (kHeadDim / 8); e += blockDim.x) {
      const int n = e % N, c = e / N;
      const int g = n / H, h = n % H;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (g < ntok)
        v = *reinterpret_cast<const uint4*>(
            p.q + (((size_t)b * p.n_q + t0 + g) * H + h) * kHeadDim + c * 8);
      *reinterpret_cast<uint4*>(qs + c * (N * 16) + n * 16) = v;
    }
    for (int e = threadIdx.x; e < G * (kHistBins / 2); e += blockDim.x) hist_s[e] = 0u;
    for (int g = 0; g < G; ++g) {
      if (g < ntok)
        load_delta(p.lse64 + ((size_t)b * p.n_q + t0 + g) * H, H, delta_s + g * H, nullptr);
      else
        for (int h = threadIdx.x; h < H; h += blockDim.x) delta_s[g * H + h] = 0.f;
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  bool ok = true;

  if (n_tiles == 0) {
    // nothing to rank in this chunk
  } else if (warp == 0) {
    // ---------------- TMA producer
    if (elect_one()) {
      const uint64_t pol = policy_evict_last();  // the other groups read the same tiles
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
      for (int i = issued > L::kStages ? issued - L::kStages : 0; i < issued; ++i)
        if (!mbar_wait(full + (i % L::kStages), (i / L::kStages) & 1)) ok = false;
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (elect_one()) {
      const uint32_t idesc = idesc_f16(128, N, true, false, false);
      const uint32_t q_addr = smem_u32(qs);
      for (int i = 0; i < n_tiles && ok; ++i) {
        const int s = i % L::kStages;
        const uint32_t ph = (i / L::kStages) & 1;
        const int buf = i & 1;
        if (!mbar_wait(full + s, ph)) { ok = false; break; }
        if (!mbar_wait(s_free + buf, ((i >> 1) & 1) ^ 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(stages + s * L::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < kHeadDim / 16; ++kk)
          mma_f16_ss(tmem_base + buf * N, kmajor_sw128_desc(a_addr, kk),
                     q_kmajor_desc<N>(q_addr, kk), idesc, kk > 0 ? 1u : 0u);
        mma_commit(s_full + buf);
        mma_commit(empty + s);
      }
      mma_commit(mma_done);
      if (!mbar_wait(mma_done, 0)) ok = false;
    }
  } else {
    // ---------------- epilogue: 128 threads, one key each, G tokens per key
    const int lg = warp & 3;
    const int t = lg * 32 + (int)lane_id();
    const float sc = p.sm_scale;
    for (int i = 0; i < n_tiles; ++i) {
      const int buf = i & 1;
      if (ok && !mbar_wait(s_full + buf, (i >> 1) & 1)) ok = false;
      tc_fence_after();
      float best[G];
#pragma unroll
      for (int g = 0; g < G; ++g) best[g] = -INFINITY;
      const uint32_t taddr = tmem_base + ((uint32_t)(lg * 32) << 16) + buf * N;
      // Four loads in flight per wait (64 columns at a time).
#pragma unroll
      for (int c0 = 0; c0 < N; c0 += 64) {
        uint32_t r[64];
#pragma unroll
        for (int c = 0; c < 64; c += 16)
          if (c0 + c < N) tmem_ld16(taddr + c0 + c, *reinterpret_cast<uint32_t(*)[16]>(r + c));
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 64; ++e)
          if (c0 + e < N)
            best[(c0 + e) / H] =
                fmaxf(best[(c0 + e) / H], __uint_as_float(r[e]) * sc - delta_s[c0 + e]);
      }
      tc_fence_before();
      mbar_arrive(s_free + buf);
      const int j = k0 + i * kKeyTile + t;
      // Per token: the key's t and one count in the token's packed histogram (plain
      // shared-memory atomics: a key's G counts go to G different histograms, and the
      // lanes of a warp spread over many bins).
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const int nc_g = nc0 + g;
        // Tokens past the group's end, or that keep all their keys, are not ranked.
        const bool valid = g < ntok && nc_g > p.k_sel && j < nc_g;
        if (valid) {
          p.tbuf[((size_t)b * p.n_q + t0 + g) * p.kv.max_len + j] = best[g];
          const uint32_t bin = ordered_key(best[g]) >> kHistShift;
          atomicAdd(hist_s + g * (kHistBins / 2) + (bin >> 1), 1u << (16 * (bin & 1)));
        }
      }
    }
    named_bar_sync(1, 128);
    for (int g = 0; g < ntok; ++g) {
      uint32_t* gh = p.hist + ((size_t)b * p.n_q + t0 + g) * kHistBins;
      for (int e = t; e < kHistBins / 2; e += 128) {
        const uint32_t w = hist_s[g * (kHistBins / 2) + e];
        if (w & 0xffffu) atomicAdd(gh + 2 * e, w & 0xffffu);
        if (w >> 16) atomicAdd(gh + 2 * e + 1, w >> 16);
      }
    }
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
static cudaError_t launch_imp_mq_t(const SelectParams& p, const CUtensorMap& tm, int batch,
                                   int n_groups, cudaStream_t st) {
  using L = ImpMqSmem<H>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(importance_mq_kernel<H>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  return launch_pdl(importance_mq_kernel<H>, dim3(p.splits2, batch * n_groups), dim3(192),
                    L::kBytes, st, tm, p, n_groups);
}

cudaError_t launch_importance_mq(const SelectParams& p, const CUtensorMap& tmap_k, int batch,
                                 cudaStream_t st) {
  if (p.chunk2 > kImpMqMaxChunk || p.chunk2 % kKeyTile != 0) return cudaErrorInvalidValue;
  const int G = kImpMqRows / p.h;
  const int n_groups = (p.n_q + G - 1) / G;
  switch (p.h) {
    case 16: return launch_imp_mq_t<16>(p, tmap_k, batch, n_groups, st);
    case 32: return launch_imp_mq_t<32>(p, tmap_k, batch, n_groups, st);
    case 48: return launch_imp_mq_t<48>(p, tmap_k, batch, n_groups, st);
    case 64: return launch_imp_mq_t<64>(p, tmap_k, batch, n_groups, st);
    case 128: return launch_imp_mq_t<128>(p, tmap_k, batch, n_groups, st);
    default: return cudaErrorInvalidValue;
  }
}

// ============================================================================
// The same pass for an FP8 E4M3 cache: raw 128-key tiles by TMA go straight into
// kind::f8f6f4 MMAs (K-major, 128-byte swizzle) against Q as two E4M3 terms
// (Q_hi + Q_lo / 16 after one power-of-two scale, exact for bf16 queries; the FP8
// full layer does the same), and each key's logits are multiplied by its k_scale.
// ============================================================================
namespace {

constexpr int kImpF8Threads = 192;  // TMA, MMA, four epilogue warps (thread = key)

template <int H>
struct ImpF8Smem {
  static constexpr int R = 8;  // raw K stages
  static constexpr uint32_t kQBytes = 2 * H * kHeadDim;  // Q_hi, Q_lo rows
  static constexpr uint32_t kRawOff = 0;
  static constexpr uint32_t kQOff = R * kE4m3TileBytes;
  static constexpr uint32_t kHistOff = kQOff + kQBytes;
  static constexpr uint32_t kDeltaOff = kHistOff + kHistBins * 4;
  static constexpr uint32_t kQinvOff = kDeltaOff + H * 4;
  static constexpr uint32_t kBarOff = kQinvOff + 16;
  static constexpr uint32_t kBars = 2 * R + 4 + 1;
  static constexpr uint32_t kSlotOff = kBarOff + kBars * 8;
  static constexpr uint32_t kBytes = kSlotOff + 16 + 1024;
  static constexpr uint32_t kTmemCols = tmem_cols_pow2(4 * H);  // two S buffers of 2H
  // (+ 2048 for the static shared memory of the Q staging and the histogram flush)
  static_assert(kBytes + 2048 <= 227 * 1024, "shared memory budget");
  static_assert(kQOff % 1024 == 0 && kBarOff % 8 == 0, "alignment");
};

}  // namespace

template <int H>
__global__ void __launch_bounds__(kImpF8Threads, 1)
    importance_fp8_kernel(const __grid_constant__ CUtensorMap tmap_k, SelectParams p) {
  using L = ImpF8Smem<H>;
  constexpr int R = L::R;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* raw = smem + L::kRawOff;
  uint8_t* qs = smem + L::kQOff;
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(smem + L::kHistOff);
  float* delta_s = reinterpret_cast<float*>(smem + L::kDeltaOff);
  float* qinv_s = reinterpret_cast<float*>(smem + L::kQinvOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* r_full = bars;
  uint64_t* r_empty = bars + R;
  uint64_t* s_full = bars + 2 * R;  // [2]
  uint64_t* s_free = s_full + 2;    // [2]
  uint64_t* mma_done = s_full + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kSlotOff);

  const int warp = threadIdx.x >> 5;
  griddep_wait();
  const int split = blockIdx.x, bq = blockIdx.y;
  const int b = bq / p.n_q, qi = bq % p.n_q;
  const int Lb = seq_len(p.kv, b, p.n_q, p.status, false);
  const int pos = Lb - p.n_q + qi;
  const int n_c = pos - p.window + 1;
  if (n_c <= p.k_sel) return;
  const int k0 = split * p.chunk2;
  const int k1 = min(k0 + p.chunk2, n_c);
  if (k0 >= k1) return;
  const int n_tiles = (k1 - k0 + kKeyTile - 1) / kKeyTile;
  const size_t row_base = (size_t)b * p.kv.max_len;

  if (threadIdx.x == 0) {
    for (int s = 0; s < R; ++s) {
      mbar_init(r_full + s, 1);
      mbar_init(r_empty + s, 1);
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
  for (int e = threadIdx.x; e < kHistBins; e += blockDim.x) hist_s[e] = 0u;
  load_delta(p.lse64 + (size_t)bq * H, H, delta_s, nullptr);
  store_q_e4m3_split<H>(qs, p.q + (size_t)bq * H * kHeadDim, qinv_s);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  bool ok = true;

  if (warp == 0) {
    if (elect_one()) {
      const uint64_t pol = policy_evict_first();
      const int row0 = (int)row_base + k0;
      int issued = 0;
      for (int i = 0; i < n_tiles && ok; ++i) {
        const int s = i % R;
        if (!mbar_wait(r_empty + s, ((i / R) & 1) ^ 1)) { ok = false; break; }
        mbar_arrive_expect_tx(r_full + s, kE4m3TileBytes);
        tma_load_2d(raw + s * kE4m3TileBytes, &tmap_k, r_full + s, 0, row0 + i * kKeyTile, pol);
        issued = i + 1;
      }
      for (int i = issued > R ? issued - R : 0; i < issued; ++i)
        if (!mbar_wait(r_full + (i % R), (i / R) & 1)) ok = false;
    }
  } else if (warp == 1) {
    if (elect_one()) {
      constexpr uint32_t idesc = idesc_e4m3(128, 2 * H, false, false);
      const uint32_t q_addr = smem_u32(qs);
      for (int i = 0; i < n_tiles && ok; ++i) {
        const int s = i % R, sb = i & 1;
        if (!mbar_wait(r_full + s, (i / R) & 1)) { ok = false; break; }
        if (!mbar_wait(s_free + sb, ((i >> 1) & 1) ^ 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(raw + s * kE4m3TileBytes);
#pragma unroll
        for (int kk = 0; kk < kHeadDim / 32; ++kk)
          mma_e4m3_ss(tmem_base + sb * 2 * H, k_e4m3_desc(a_addr, kk),
                      q_e4m3_desc<2 * H>(q_addr, kk), idesc, kk > 0 ? 1u : 0u);
        mma_commit(s_full + sb);
        mma_commit(r_empty + s);
      }
      mma_commit(mma_done);
      if (!mbar_wait(mma_done, 0)) ok = false;
    }
  } else {
    // epilogue: thread t owns key t of the tile
    const int lg = warp & 3;
    const int t = lg * 32 + (int)lane_id();
    float* trow = p.tbuf + (size_t)bq * p.kv.max_len;
    const float qsc = qinv_s[0] * p.sm_scale;  // Q-scaled logit -> s (before k_scale)
    auto scale_of = [&](int i) {
      const int j = k0 + i * kKeyTile + t;
      return (i < n_tiles && j < k1) ? __ldg(p.kv.k_scale + row_base + j) : 0.f;
    };
    float ks_next = scale_of(0), ks_far = scale_of(1);
    for (int i = 0; i < n_tiles; ++i) {
      const int buf = i & 1;
      const float m = qsc * ks_next;
      ks_next = ks_far;
      ks_far = scale_of(i + 2);
      if (ok && !mbar_wait(s_full + buf, (i >> 1) & 1)) ok = false;
      tc_fence_after();
      float best = -INFINITY;
      const uint32_t taddr = tmem_base + ((uint32_t)(lg * 32) << 16) + buf * 2 * H;
#pragma unroll
      for (int c0 = 0; c0 < H; c0 += 32) {  // hi and lo of 32 heads: four loads per wait
        uint32_t r[64];
#pragma unroll
        for (int c = 0; c < 32; c += 16)
          if (c0 + c < H) {
            tmem_ld16(taddr + c0 + c, *reinterpret_cast<uint32_t(*)[16]>(r + c));
            tmem_ld16(taddr + H + c0 + c, *reinterpret_cast<uint32_t(*)[16]>(r + 32 + c));
          }
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (c0 + e < H) {
            const float x = fmaf(__uint_as_float(r[32 + e]), 0.0625f, __uint_as_float(r[e]));
            best = fmaxf(best, x * m - delta_s[c0 + e]);
          }
      }
      tc_fence_before();
      mbar_arrive(s_free + buf);
      const int j = k0 + i * kKeyTile + t;
      const bool valid = j < k1;
      if (valid) trow[j] = best;
      if (valid) atomicAdd(hist_s + (ordered_key(best) >> kHistShift), 1u);
    }
    named_bar_sync(1, 128);
    __shared__ uint32_t flush_red[128 + 1];
    flush_hist_top<128>(hist_s, p.hist + (size_t)bq * kHistBins, p.k_sel, t, flush_red,
                        [] { named_bar_sync(1, 128); });
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
static cudaError_t launch_imp_f8_t(const SelectParams& p, const CUtensorMap& tm, int bq,
                                   cudaStream_t st) {
  using L = ImpF8Smem<H>;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(importance_fp8_kernel<H>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  return launch_pdl(importance_fp8_kernel<H>, dim3(p.splits2, bq), dim3(kImpF8Threads), L::kBytes,
                    st, tm, p);
}

cudaError_t launch_importance_fp8(const SelectParams& p, const CUtensorMap& tmap_k, int bq,
                                  cudaStream_t st) {
  switch (p.h) {
    case 16: return launch_imp_f8_t<16>(p, tmap_k, bq, st);
    case 32: return launch_imp_f8_t<32>(p, tmap_k, bq, st);
    case 48: return launch_imp_f8_t<48>(p, tmap_k, bq, st);
    case 64: return launch_imp_f8_t<64>(p, tmap_k, bq, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace hs2
