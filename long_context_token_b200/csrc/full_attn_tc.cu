// Full-attention layer on the 5th-generation tensor cores (bf16 cache, h_q <= 64).
//
// Split-K flash-decode of the hybrid block's full layer (toolnavs article 2080, fr
// "Ce que fait HySparse2": the full layer attends over the whole context; MQA per
// "Les chiffres mesurés").  One CTA per key chunk of one (sequence, query token):
//
//   warp 0      TMA producer: 128-key K and V tiles (two 64-column boxes each,
//               128-byte swizzle) into an NS-stage ring, K and V on separate
//               barriers;
//   warp 1      TMEM allocator, MMA issuer:
//                 S^T[128 keys x H] = K_tile . Q^T          (8 x K=16, TMEM ping-pong)
//                 O^T[128 d x H]  += V_tile^T . (P_hi + P_lo)^T  (16 x K=16)
//               the P.V of tile i-1 is issued after the Q.K of tile i;
//   warps 2..5  softmax: thread t owns key t of the tile (TMEM lane t).  Logits go to
//               the log2 domain, x = s * sm_scale * log2(e) - m_h; the per-head
//               reference m_h only moves when some x exceeds 8 (then the tile max
//               is taken across the 128 threads and O is rescaled in TMEM), so the
//               common tile needs no cross-thread reduction.  p = 2^x is split into
//               bf16 hi + lo so that P.V keeps ~16 bits of p; per-thread partial
//               sums l_h are reduced once at the end of the chunk.
// Each CTA writes its chunk's partial (m in log2 units, l, unnormalised o); merge.cu
// combines the chunks.
#include <cuda_bf16.h>
#include <string.h>

#include "hs2_internal.cuh"
#include "sm100.cuh"
#include "tc_common.cuh"
#include "decode_select.cuh"

namespace hs2 {

using namespace sm100;

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleAt = 8.0f;  // log2 units: move the reference when p would exceed 2^8

// Gather mode (a sparse layer) keeps one stage: its CTAs mostly take a single tile, and
// the smaller footprint lets two CTAs share an SM.
template <int H, bool GATHER>
struct FullSmem {
  static constexpr int kStages = GATHER ? 1 : (H <= 16 ? 3 : 2);
  static constexpr uint32_t kTile = kKTileBytesBf16;    // one K or V tile
  static constexpr uint32_t kQBytes = H * kHeadDim * 2;
  static constexpr uint32_t kPBytes = kKeyTile * H * 2;  // one of hi / lo
  static constexpr uint32_t kKOff = 0;
  static constexpr uint32_t kVOff = kStages * kTile;
  static constexpr uint32_t kQOff = 2 * kStages * kTile;
  static constexpr uint32_t kPOff = kQOff + kQBytes;        // [2 buffers][hi, lo]
  static constexpr uint32_t kRedOff = kPOff + 4 * kPBytes;  // [4 warps][H] floats
  static constexpr uint32_t kRefOff = kRedOff + 4 * H * 4;  // [H] reference, [H] alpha
  static constexpr uint32_t kBarOff = kRefOff + 2 * H * 4;
  static constexpr uint32_t kBars = 4 * kStages + 10 + kTileRing;
  static constexpr uint32_t kSlotOff = kBarOff + kBars * 8;
  static constexpr uint32_t kRingOff = kSlotOff + 16;  // [kTileRing] tile indices
  // Histogram of the selection bounds u (full layer only).
  static constexpr uint32_t kUHistOff = (kRingOff + 4 * kTileRing + 15) / 16 * 16;
  static constexpr uint32_t kUHistLen = GATHER ? 0u : hs2::kUHistBytes;
  static constexpr uint32_t kBytes = kUHistOff + kUHistLen + 1024;
  static constexpr uint32_t kTmemCols = tmem_cols_pow2(3 * H);
  static_assert(kBytes <= 227 * 1024, "shared memory budget");
};

// Largest value of v over the 128 softmax threads, per head (named barrier 1).
template <int H>
__device__ __forceinline__ void block_max_heads(const float (&v)[H], float* red, float* out,
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

// Fused tail of the full layer (decode_select.cuh): the CTAs of a row merge their
// partials and (fuse 2) select the row's tokens, in the K/V stages, idle by now.  A
// function of its own, called after the stream: every index is recomputed here from the
// CTA's coordinates and the parameters, so that nothing stays live in registers across
// the stream for it.  Candidates' K rows are gathered into the first stages and go through
// the stream's S^T = K . Q^T MMA (S buffers at TMEM columns [tile H, tile H + H)).
template <int H>
__device__ __noinline__ bool full_tc_tail(const FullParams& p) {
  using L = FullSmem<H, false>;
  constexpr int NS = L::kStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  const uint32_t k_addr = smem_u32(smem + L::kKOff);
  const uint8_t* qs = smem + L::kQOff;
  const uint32_t q_addr = smem_u32(qs);
  uint64_t* post_bar = reinterpret_cast<uint64_t*>(smem + L::kBarOff) + 4 * NS + 9;
  const uint32_t* tmem_slot = reinterpret_cast<const uint32_t*>(smem + L::kSlotOff);
  const uint32_t* uhist_s = reinterpret_cast<const uint32_t*>(smem + L::kUHistOff);
  const int warp = threadIdx.x >> 5;
  const int split = blockIdx.x, bq = blockIdx.y;
  const int b = bq / p.n_q, qi = bq % p.n_q;
  const int pos = seq_len(p.kv, b, p.n_q, p.status, false) - p.n_q + qi;
  const int k0 = split * p.chunk1;
  const int k1 = min(k0 + p.chunk1, pos + 1);
  const size_t row_base = (size_t)b * p.kv.max_len;
  const float c2 = p.sm_scale * kLog2e;
  auto recompute = [&](const int* list, int m, float* t2, uint32_t round, const float* D) -> bool {
    bool rok = true;
    const int ntile = (m + kKeyTile - 1) / kKeyTile;
    for (int tl = 0; tl < ntile; ++tl)
      gather_list_rows<16, kBoxBytes>(k_addr + tl * L::kTile, static_cast<const uint8_t*>(p.kv.k),
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
        const uint32_t id_qk = idesc_f16(128, H, true, false, false);
        for (int tl = 0; tl < ntile; ++tl) {
#pragma unroll
          for (int kk = 0; kk < kHeadDim / 16; ++kk)
            mma_f16_ss(tmem_base + tl * H, kmajor_sw128_desc(k_addr + tl * L::kTile, kk),
                       q_kmajor_desc<H>(q_addr, kk), id_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(post_bar);
      }
      __syncwarp();
    } else if (warp >= 2) {
      const int lg = warp & 3;
      const int t = lg * 32 + (int)lane_id();
      const uint32_t lane_base = (uint32_t)(lg * 32) << 16;
      if (!mbar_wait(post_bar, round & 1u)) rok = false;
      tc_fence_after();
      for (int tl = 0; tl < ntile; ++tl) {
        uint32_t r[H];
#pragma unroll
        for (int c = 0; c < H; c += 16)
          tmem_ld16(tmem_base + lane_base + tl * H + c, *reinterpret_cast<uint32_t(*)[16]>(r + c));
        tmem_wait_ld();
        const int slot = tl * kKeyTile + t;
        if (slot < m) {
          float v = -INFINITY;
#pragma unroll
          for (int h = 0; h < H; ++h) v = fmaxf(v, __uint_as_float(r[h]) * c2 - D[h]);
          t2[slot] = v;
        }
      }
      tc_fence_before();
    }
    __syncthreads();
    return rok;
  };
  QView qv;
  qv.base = qs;         // Q as the MMA's K-major operand: chunk c of head h at
  qv.hstride = 16;      // c * H * 16 + h * 16
  qv.cstride = H * 16;
  // The partial's m per head is still in the softmax warps' reference array, unless the
  // CTA took no tile (the same rule as the stream's).
  const bool dyn = p.splits1 > 1 && !p.deterministic;
  const bool took = dyn ? split < (pos + kKeyTile) / kKeyTile : k0 < k1;
  const float* own_m = took ? reinterpret_cast<const float*>(smem + L::kRefOff) : nullptr;
  return fused_tail<H, false, 6>(p, smem, 2u * NS * L::kTile, L::kTile, uhist_s, own_m, bq, b,
                                 split, pos, k0, k1, qv, recompute);
}

template <int H, bool GATHER>
__global__ void __launch_bounds__(192, (GATHER && H <= 16) ? 2 : 1)
    full_attn_tc_kernel(const __grid_constant__ CUtensorMap tmap_k,
                        const __grid_constant__ CUtensorMap tmap_v,
                        const __grid_constant__ FullParams p) {
  using L = FullSmem<H, GATHER>;
  constexpr int NS = L::kStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* kst = smem + L::kKOff;
  uint8_t* vst = smem + L::kVOff;
  uint8_t* qs = smem + L::kQOff;
  uint8_t* ps = smem + L::kPOff;
  float* red = reinterpret_cast<float*>(smem + L::kRedOff);
  float* mref_s = reinterpret_cast<float*>(smem + L::kRefOff);
  float* alpha_s = mref_s + H;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* kfull = bars;
  uint64_t* kempty = bars + NS;
  uint64_t* vfull = bars + 2 * NS;
  uint64_t* vempty = bars + 3 * NS;
  uint64_t* s_full = bars + 4 * NS;      // [2]
  uint64_t* s_free = s_full + 2;         // [2]
  uint64_t* p_full = s_full + 4;         // [2]
  uint64_t* p_free = s_full + 6;         // [2]
  uint64_t* mma_done = s_full + 8;
  uint64_t* post_bar = s_full + 9;  // MMAs of the selection tail
  uint64_t* idx_bar = s_full + 10;  // [kTileRing] one per slot of the tile-index ring
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kSlotOff);
  int* tile_ring = reinterpret_cast<int*>(smem + L::kRingOff);
  uint32_t* uhist_s = reinterpret_cast<uint32_t*>(smem + L::kUHistOff);

  const int warp = threadIdx.x >> 5;
  const int split = blockIdx.x, bq = blockIdx.y;
  const int b = bq / p.n_q, qi = bq % p.n_q;

  // Set-up that touches no global memory, overlapping the previous kernel's tail.
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(kfull + s, GATHER ? 32 : 1);
      mbar_init(kempty + s, 1);
      mbar_init(vfull + s, GATHER ? 32 : 1);
      mbar_init(vempty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(s_full + s, 1);
      mbar_init(s_free + s, 128);
      mbar_init(p_full + s, 128);
      mbar_init(p_free + s, 1);
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
  // A sparse layer (gather mode with the on-chip merge) reads nothing that the previous
  // kernel of this library writes before letting its dependents start (the selection
  // publishes the index set first; a sparse layer writes only its own output): it waits
  // for the previous grid only before writing its output, so its gathers overlap the
  // previous kernel's tail.  Index entries are read through L2.
  const bool defer_wait = GATHER && p.out != nullptr;
  if (!defer_wait) griddep_wait();
  // A sparse layer lets the next kernel start at once: the next sparse layer needs
  // nothing from this one and, like this one, waits before writing its output; every
  // other kernel of the library waits for this grid to end before it reads anything.
  if (defer_wait) griddep_launch_dependents();

  const int Lb = seq_len(p.kv, b, p.n_q, p.status, !GATHER && split == 0 && qi == 0);
  const int pos = Lb - p.n_q + qi;
  // Keys [k0, k1) of the sequence, or (gather mode) index entries [k0, k1) of the row.
  const int k0 = split * p.chunk1;
  const int k1 = GATHER ? min(k0 + p.chunk1, p.idx_width) : min(k0 + p.chunk1, pos + 1);
  const int32_t* idx_row = GATHER ? p.idx + (size_t)bq * p.idx_width : nullptr;
  const size_t row_base = (size_t)b * p.kv.max_len;
  // Fused full layer with several CTAs a row: the row's tiles are shared out at run time
  // (CTA r takes tiles r, r + S, ..., r + (NS - 1) S, then claims the next free tile
  // from the row's counter until none is left), so that CTAs slowed by the memory
  // system take fewer tiles and the row's CTAs reach its first barrier together.  The
  // selection keeps its static ownership of positions (chunk r), whoever read them.
  const int S = p.splits1;
  const bool dyn = !GATHER && p.fuse != 0 && S > 1 && !p.deterministic;
  const int row_tiles = (pos + 1 + kKeyTile - 1) / kKeyTile;
  const int n_tiles = dyn ? (split < row_tiles ? 1 : 0)  // (only whether any)
                          : (k0 < k1 ? (k1 - k0 + kKeyTile - 1) / kKeyTile : 0);
  const int k_end = dyn ? pos + 1 : k1;  // keys at or past this one are masked
  const size_t pidx = (size_t)bq * p.splits1 + split;
  // Cluster mode keeps the partial in this CTA's shared memory (the K stages, idle by
  // the time the partial is written) for the on-chip merge.
  const bool on_chip = GATHER && p.out != nullptr;
  float* part_o = on_chip ? reinterpret_cast<float*>(smem + kClusterOOff)
                          : p.part_o + pidx * H * kHeadDim;
  float* part_ml = on_chip ? reinterpret_cast<float*>(smem + kClusterMlOff)
                           : p.part_ml + pidx * H * 2;
  bool ok = true;

  if (n_tiles == 0) {
    // Empty chunk: an empty partial (no key).
    for (int h = threadIdx.x; h < H; h += blockDim.x) {
      part_ml[2 * h] = -INFINITY;
      part_ml[2 * h + 1] = 0.f;
    }
  } else {
    if (GATHER) {
      // The first tile's rows are gathered by every thread of the CTA (the issue of
      // 4096 16-byte copies is the gather's cost); warp 0 gathers any later tiles.
      gather_tile_rows<16, kBoxBytes>(smem_u32(kst), smem_u32(vst),
                                      static_cast<const uint8_t*>(p.kv.k),
                                      static_cast<const uint8_t*>(p.kv.v), idx_row, k0, k1, Lb,
                                      row_base, p.status, threadIdx.x, blockDim.x);
    }
    store_q_kmajor<H>(qs, p.q + (size_t)bq * H * kHeadDim, threadIdx.x, blockDim.x);
    if (GATHER) cp_async_wait_all();
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const uint32_t tmem_o = tmem_base + 2 * H;

    if (GATHER && warp == 0) {
      // ------------------------------------------------ gather producer (32 lanes)
      // Rows named by the index row go to the same 128-byte-swizzled layout that TMA
      // writes (16-byte chunk c of row r at chunk c ^ (r mod 8)); absent rows are
      // zero-filled.  Each lane copies 4 rows, waits for its copies and arrives.
      // K and V of a later tile are gathered on their own barriers: with one stage the
      // P.V of tile i-1 (which frees V) is issued only after the Q.K of tile i.
      const int lane = (int)lane_id();
      const uint8_t* kb = static_cast<const uint8_t*>(p.kv.k);
      const uint8_t* vb = static_cast<const uint8_t*>(p.kv.v);
      for (int i = 0; i < n_tiles; ++i) {
        const int s = i % NS;
        const uint32_t ph = ((i / NS) & 1) ^ 1;
        if (i > 0) {  // tile 0 was gathered by the whole CTA above
          if (ok && !mbar_wait(kempty + s, ph)) ok = false;
          gather_tile_rows<16, kBoxBytes>(smem_u32(kst + s * L::kTile), 0u, kb, nullptr, idx_row,
                                          k0 + i * kKeyTile, k1, Lb, row_base, p.status, lane,
                                          32);
          cp_async_wait_all();
          fence_proxy_async_smem();
        }
        mbar_arrive(kfull + s);
        if (i > 0) {
          if (ok && !mbar_wait(vempty + s, ph)) ok = false;
          gather_tile_rows<16, kBoxBytes>(0u, smem_u32(vst + s * L::kTile), nullptr, vb, idx_row,
                                          k0 + i * kKeyTile, k1, Lb, row_base, p.status, lane,
                                          32);
          cp_async_wait_all();
          fence_proxy_async_smem();
        }
        mbar_arrive(vfull + s);
      }
    } else if (warp == 0) {
      // ------------------------------------------------------------ TMA producer
      if (elect_one()) {
        // Tile i's index goes to slot i of the ring (its barrier arrived on) before the
        // tile's loads; past the last tile an index of -1 ends the MMA warp's and the
        // softmax warps' loops.  (The stage barriers see loads only: their phases stay in
        // step with the tiles, which the wait for the last loads below relies on.)
        const uint64_t pol = policy_evict_first();
        const int row_b = b * p.kv.max_len;
        uint32_t* row_counter = p.rowsync + (size_t)bq * 8 + kRowTileSlot;
        uint32_t claimed = 0;
        int issued = 0;
        const bool stall = p.stall_test == 1;  // the stall test issues no load
        for (int i = 0; ok && !stall; ++i) {
          const int s = i % NS;
          const uint32_t ph = ((i / NS) & 1) ^ 1;
          const int tile = dyn ? (i < NS ? split + i * S : NS * S + (int)claimed)
                               : (i < n_tiles ? k0 / kKeyTile + i : -1);
          const bool end = tile < 0 || tile >= row_tiles || (!dyn && i >= n_tiles);
          if (!mbar_wait(kempty + s, ph)) { ok = false; break; }
          tile_ring[i % kTileRing] = end ? -1 : tile;
          mbar_arrive(idx_bar + i % kTileRing);
          if (end) break;
          if (dyn && i + 1 >= NS) claimed = atomicAdd(row_counter, 1u);  // tile i + 1's
          const int row = row_b + tile * kKeyTile;
          mbar_arrive_expect_tx(kfull + s, L::kTile);
          tma_load_2d(kst + s * L::kTile, &tmap_k, kfull + s, 0, row, pol);
          tma_load_2d(kst + s * L::kTile + kBoxBytes, &tmap_k, kfull + s, 64, row, pol);
          if (!mbar_wait(vempty + s, ph)) { ok = false; break; }
          mbar_arrive_expect_tx(vfull + s, L::kTile);
          tma_load_2d(vst + s * L::kTile, &tmap_v, vfull + s, 0, row, pol);
          tma_load_2d(vst + s * L::kTile + kBoxBytes, &tmap_v, vfull + s, 64, row, pol);
          issued = i + 1;
        }
        for (int i = issued > NS ? issued - NS : 0; i < issued; ++i) {
          if (!mbar_wait(kfull + (i % NS), (i / NS) & 1)) ok = false;
          if (!mbar_wait(vfull + (i % NS), (i / NS) & 1)) ok = false;
        }
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      if (elect_one()) {
        const uint32_t id_qk = idesc_f16(128, H, true, false, false);
        const uint32_t id_pv = idesc_f16(128, H, true, true, true);
        const uint32_t q_addr = smem_u32(qs);
        auto issue_pv = [&](int t) -> bool {
          const int s = t % NS, pb = t & 1;
          if (!mbar_wait(vfull + s, (t / NS) & 1)) return false;
          if (!mbar_wait(p_full + pb, (t >> 1) & 1)) return false;
          tc_fence_after();
          const uint32_t v_addr = smem_u32(vst + s * L::kTile);
          const uint32_t p_hi = smem_u32(ps + (2 * pb) * L::kPBytes);
          const uint32_t p_lo = p_hi + L::kPBytes;
#pragma unroll
          for (int kk = 0; kk < kKeyTile / 16; ++kk)
            mma_f16_ss(tmem_o, vt_mnmajor_sw128_desc(v_addr, kk), pt_mnmajor_desc(p_hi, kk),
                       id_pv, (t > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < kKeyTile / 16; ++kk)
            mma_f16_ss(tmem_o, vt_mnmajor_sw128_desc(v_addr, kk), pt_mnmajor_desc(p_lo, kk),
                       id_pv, 1u);
          mma_commit(p_free + pb);
          mma_commit(vempty + s);
          return true;
        };
        if (!GATHER && p.stall_test == 1) ok = false;  // the stall test issues no MMA
        int n_done = 0;
        for (int i = 0; (GATHER ? i < n_tiles : true) && ok; ++i) {
          const int s = i % NS, sb = i & 1;
          if (!GATHER) {  // the tile's index first (-1: past the last tile)
            if (!mbar_wait(idx_bar + i % kTileRing, (i / kTileRing) & 1)) { ok = false; break; }
            if (tile_ring[i % kTileRing] < 0) break;
          }
          if (!mbar_wait(kfull + s, (i / NS) & 1)) { ok = false; break; }
          n_done = i + 1;
          if (!mbar_wait(s_free + sb, ((i >> 1) & 1) ^ 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t k_addr = smem_u32(kst + s * L::kTile);
#pragma unroll
          for (int kk = 0; kk < kHeadDim / 16; ++kk)
            mma_f16_ss(tmem_base + sb * H, kmajor_sw128_desc(k_addr, kk),
                       q_kmajor_desc<H>(q_addr, kk), id_qk, kk > 0 ? 1u : 0u);
          mma_commit(s_full + sb);
          mma_commit(kempty + s);
          if (i > 0 && !issue_pv(i - 1)) { ok = false; break; }
        }
        if (ok && n_done > 0 && !issue_pv(n_done - 1)) ok = false;
        mma_commit(mma_done);
        if (!mbar_wait(mma_done, 0)) ok = false;
      }
    } else {
      // ------------------------------------------------------------ softmax
      const int lg = warp & 3;
      const int t = lg * 32 + (int)lane_id();  // key of the tile == TMEM lane
      const uint32_t lane_base = (uint32_t)(lg * 32) << 16;
      const float c2 = p.sm_scale * kLog2e;
      const uint64_t keep_policy = policy_evict_last();
      // Fused selection: keys [0, n_c) record their bound u_j = max_h x_hj and count it.
      const int n_c = pos - p.window + 1;
      const bool sel_keys = !GATHER && p.fuse == 2 && n_c > p.k_sel;
      float* urow = sel_keys ? p.ubuf + (size_t)bq * p.ld_u : nullptr;
      float l[H];
#pragma unroll
      for (int h = 0; h < H; ++h) l[h] = 0.f;
      if (t < H) mref_s[t] = -INFINITY;
      named_bar_sync(1, 128);
      int n_done = 0;
      for (int i = 0; GATHER ? i < n_tiles : true; ++i) {
        // A failed wait in any softmax thread stops the waits of all of them (they
        // keep taking part in the named barriers, so none is left behind).  Without
        // gathers the tile comes from the producer's ring (-1: no more tiles).
        const int sb = i & 1;
        int tile = k0 / kKeyTile + i;
        if (!GATHER) {
          const long long limit = p.stall_test == 1 ? kStallTestCycles : kWaitCycles;
          if (ok && !mbar_wait(idx_bar + i % kTileRing, (i / kTileRing) & 1, limit)) ok = false;
          tile = ok ? tile_ring[i % kTileRing] : -1;
          if (named_bar_or(3, 128, !ok)) ok = false;
          if (!ok || tile < 0) break;  // the same for every softmax thread
        }
        n_done = i + 1;
        if (ok && !mbar_wait(s_full + sb, (i >> 1) & 1)) ok = false;
        if (named_bar_or(3, 128, !ok)) ok = false;
        tc_fence_after();
        float x[H];
        {
          // Every chunk's load in flight before the one wait.
          uint32_t r[H];
#pragma unroll
          for (int c = 0; c < H; c += 16)
            tmem_ld16(tmem_base + lane_base + sb * H + c, *reinterpret_cast<uint32_t(*)[16]>(r + c));
          tmem_wait_ld();
          if (!GATHER && p.sbuf) {
            // Raw float32 logits of keys outside the window, for the selection (kept in
            // L2 with an evict-last policy; the selection reads them right after).
            const int jj = tile * kKeyTile + t;
            if (jj < k_end && jj <= pos - p.window && pos - p.window + 1 > p.k_sel) {
              float* dst = p.sbuf + ((size_t)bq * p.kv.max_len + jj) * H;
#pragma unroll
              for (int e = 0; e < H / 4; ++e)
                st_global_v4_hint(dst + 4 * e,
                                  make_uint4(r[4 * e], r[4 * e + 1], r[4 * e + 2], r[4 * e + 3]),
                                  keep_policy);
            }
          }
#pragma unroll
          for (int e = 0; e < H; ++e) x[e] = __uint_as_float(r[e]) * c2;
        }
        tc_fence_before();
        mbar_arrive(s_free + sb);
        const int j = tile * kKeyTile + t;
        bool valid = j < k_end;
        if (sel_keys && valid && j < n_c) {
          float u = x[0];
#pragma unroll
          for (int h = 1; h < H; ++h) u = fmaxf(u, x[h]);
          st_global_f32_hint(urow + j, u, keep_policy);
          atomicAdd(&uhist_s[ubin(u)], 1u);
        }
        if (GATHER && valid) {
          const int pj = __ldcg(idx_row + j);
          valid = pj >= 0 && pj < Lb;
        }
        bool over = false;
#pragma unroll
        for (int h = 0; h < H; ++h) {
          if (!valid) x[h] = -INFINITY;
          over |= x[h] - mref_s[h] > kRescaleAt;
        }
        if (named_bar_or(2, 128, over)) {
          // New per-head reference: the larger of the old one and this tile's max.
          block_max_heads<H>(x, red, alpha_s, t);
          if (t < H) {
            const float mnew = fmaxf(mref_s[t], alpha_s[t]);
            alpha_s[t] = exp2f(mref_s[t] - mnew);  // 0 on the first tile
            mref_s[t] = mnew;
          }
          named_bar_sync(1, 128);
#pragma unroll
          for (int h = 0; h < H; ++h) l[h] *= alpha_s[h];
          if (i > 0) {
            // O holds the P.V of tiles < i: wait for the last one, then rescale.
            if (ok && !mbar_wait(p_free + ((i - 1) & 1), ((i - 1) >> 1) & 1)) ok = false;
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < H; c += 16) {
              uint32_t r[16];
              tmem_ld16(tmem_o + lane_base + c, r);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 16; ++e)
                r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha_s[c + e]);
              tmem_st16(tmem_o + lane_base + c, r);
            }
            tmem_wait_st();
            tc_fence_before();
          }
        }
        // P for this tile into buffer sb (free once the P.V of tile i-2 is done).
        if (ok && i >= 2 && !mbar_wait(p_free + sb, ((i >> 1) & 1) ^ 1)) ok = false;
        uint8_t* phi = ps + (2 * sb) * L::kPBytes;
        uint8_t* plo = phi + L::kPBytes;
#pragma unroll
        for (int c = 0; c < H / 8; ++c) {
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int h0 = c * 8 + 2 * e;
            // A head whose reference is still -inf has seen no key: its p is 0 (not
            // 2^(-inf - -inf)), so a leading all-padding tile leaves O and l at zero.
            const float p0 = ex2_ftz(x[h0] - finite_ref(mref_s[h0]));
            const float p1 = ex2_ftz(x[h0 + 1] - finite_ref(mref_s[h0 + 1]));
            l[h0] += p0;
            l[h0 + 1] += p1;
            split_bf16_hi_lo(p0, p1, hw[e], lw[e]);
          }
          *reinterpret_cast<uint4*>(phi + c * (kKeyTile * 16) + t * 16) =
              make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(plo + c * (kKeyTile * 16) + t * 16) =
              make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
        if (!GATHER && !valid) {
          // Rows past the row's end (only its last tile has them) may hold anything, NaN
          // included; 0 * NaN would poison P.V, so zero this key's V row once its tile
          // has landed.
          const int s = i % NS;
          if (ok && !mbar_wait(vfull + s, (i / NS) & 1)) ok = false;
          uint4* v0 = reinterpret_cast<uint4*>(vst + s * L::kTile + t * 128);
          uint4* v1 = reinterpret_cast<uint4*>(vst + s * L::kTile + kBoxBytes + t * 128);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            v0[e] = make_uint4(0, 0, 0, 0);
            v1[e] = make_uint4(0, 0, 0, 0);
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(p_full + sb);
      }
      // The merge kernel may be scheduled (it waits for this grid); with the fused tail the
      // next kernel starts only once the index set is written.
      if (GATHER || !p.fuse) griddep_launch_dependents();
      // Epilogue: O^T row t is dimension t of every head; l is reduced across threads.
      const int last = n_done - 1;
      if (ok && n_done > 0 && !mbar_wait(p_free + (last & 1), (last >> 1) & 1)) ok = false;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < H; c += 16) {
        uint32_t r[16];
        tmem_ld16(tmem_o + lane_base + c, r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) part_o[(c + e) * kHeadDim + t] = __uint_as_float(r[e]);
      }
      tc_fence_before();
#pragma unroll
      for (int h = 0; h < H; ++h) {
        const float s = warp_sum(l[h]);
        if (lane_id() == 0) red[(warp & 3) * H + h] = s;
      }
      named_bar_sync(1, 128);
      if (t < H) {
        part_ml[2 * t] = mref_s[t];
        part_ml[2 * t + 1] = red[t] + red[H + t] + red[2 * H + t] + red[3 * H + t];
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
    if (p.fuse && !full_tc_tail<H>(p)) set_status(p.status, HS2_ERR_DEVICE_TIMEOUT);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(*tmem_slot, L::kTmemCols);
  }
}

template <int H, bool GATHER>
static cudaError_t launch_full_tc_t(FullParams p, const CUtensorMap& tk, const CUtensorMap& tv,
                                    int bq, cudaStream_t st) {
  using L = FullSmem<H, GATHER>;
  auto kernel = full_attn_tc_kernel<H, GATHER>;
  static int max_cluster = 0;
  if (!max_cluster) {
    cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
    if (e != cudaSuccess) return e;
    max_cluster = GATHER ? largest_cluster(kernel, dim3(192), L::kBytes) : 1;
    if (max_cluster < 1) return cudaErrorLaunchOutOfResources;
  }
  if (!GATHER)
    return launch_pdl_coop(kernel, dim3(p.splits1, bq), dim3(192), L::kBytes,
                           p.fuse != 0 && p.splits1 > 1, st, tk, tv, p);
  plan_gather_cluster(p.idx_width, max_cluster, &p.splits1, &p.chunk1);
  return launch_pdl_cluster(kernel, dim3(p.splits1, bq), dim3(192), L::kBytes, p.splits1, st, tk,
                            tv, p);
}

template <bool GATHER>
static cudaError_t launch_full_tc_h(const FullParams& p, const CUtensorMap& tk,
                                    const CUtensorMap& tv, int bq, cudaStream_t st) {
  switch (p.h) {
    case 16: return launch_full_tc_t<16, GATHER>(p, tk, tv, bq, st);
    case 32: return launch_full_tc_t<32, GATHER>(p, tk, tv, bq, st);
    case 48: return launch_full_tc_t<48, GATHER>(p, tk, tv, bq, st);
    case 64: return launch_full_tc_t<64, GATHER>(p, tk, tv, bq, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_full_attn_tc(const FullParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                                int bq, cudaStream_t st) {
  return launch_full_tc_h<false>(p, tk, tv, bq, st);
}

cudaError_t launch_sparse_attn_tc(FullParams p, int bq, cudaStream_t st) {
  CUtensorMap unused;
  memset(&unused, 0, sizeof(unused));
  return launch_full_tc_h<true>(p, unused, unused, bq, st);
}

}  // namespace hs2
