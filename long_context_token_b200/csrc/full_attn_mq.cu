// Full-attention layer for several new tokens of a sequence at once (KV append, bf16
// cache) on the 5th-generation tensor cores.
//
// Same method as the one-token decode (toolnavs article 2080, fr "Ce que fait
// HySparse2": the full layer attends over the whole context; one shared K/V head per
// "Les chiffres mesurés"), with the causal rule of appended tokens: token i of n_q sits
// at p = L - n_q + i and sees keys [0, p].  Here the MMA's M is the 128 query rows
// (G = 128 / H tokens x H heads of one sequence), so every K/V tile brought on chip
// serves G tokens at once:
//
//   S[128 rows x 64 keys]  = Q . K_tile^T                (8 x K=16, TMEM ping-pong)
//   O[128 rows x 128 d]   += (P_hi + P_lo) . V_tile       (2 x 4 x K=16)
//
//   warp 0      TMA producer: 64-key K and V tiles (two 64-column boxes, 128-byte
//               swizzle) into a 3-stage ring;
//   warp 1      TMEM allocator, MMA issuer (the P.V of tile i-1 after the Q.K of i);
//   warps 2..9  softmax: query row r (TMEM lane r) is owned by two threads, of warps
//               w and w + 4, each taking 32 of the tile's 64 keys and half of the
//               row of O; they exchange their tile maxima through shared memory.
//               Logits go to the log2 domain; the row's reference only moves when a
//               logit exceeds it by more than 8 (then the row of O is rescaled in
//               TMEM); p = 2^(x - m) is split into bf16 hi + lo so that P.V keeps
//               ~16 bits of p.
// Each CTA writes the partial (m in log2 units, l, unnormalised o) of each of its rows
// for its key chunk, in the layout of the one-token kernel; merge.cu combines them.
#include <cuda_bf16.h>
#include <string.h>

#include "hs2_internal.cuh"
#include "sm100.cuh"
#include "tc_common.cuh"

namespace hs2 {

using namespace sm100;

namespace {

constexpr float kLog2eMq = 1.4426950408889634f;
constexpr float kRescaleAtMq = 8.0f;
constexpr int kMqRows = 128;                  // query rows per CTA (the MMA's M)
constexpr int kMqKeys = 64;                   // keys per tile
constexpr uint32_t kMqBox = kMqKeys * 128;    // 64 rows x 128 B: one swizzled box
constexpr uint32_t kMqTile = 2 * kMqBox;      // 64 keys x 128 d x bf16

constexpr int kMqSoftmax = 256;                 // softmax threads (two per query row)
constexpr int kMqThreads = 64 + kMqSoftmax;

struct MqSmem {
  static constexpr int kStages = 3;
  static constexpr uint32_t kKOff = 0;
  static constexpr uint32_t kVOff = kStages * kMqTile;
  static constexpr uint32_t kQOff = 2 * kStages * kMqTile;
  static constexpr uint32_t kQBytes = kMqRows * kHeadDim * 2;
  static constexpr uint32_t kPBytes = kMqRows * kMqKeys * 2;  // one of hi / lo
  static constexpr uint32_t kPOff = kQOff + kQBytes;           // [2 buffers][hi, lo]
  static constexpr uint32_t kRedOff = kPOff + 4 * kPBytes;     // [2 tiles][2 halves][128] f32
  static constexpr uint32_t kBarOff = kRedOff + 2 * 2 * kMqRows * 4;
  static constexpr uint32_t kBars = 4 * kStages + 9;
  static constexpr uint32_t kSlotOff = kBarOff + kBars * 8;
  static constexpr uint32_t kBytes = kSlotOff + 16 + 1024;
  static constexpr uint32_t kTmemCols = 256;  // S ping-pong (2 x 64) + O (128)
  static_assert(kBytes <= 227 * 1024, "shared memory budget");
};

// A operand Q or P (rows x K, K-major, unswizzled, [K/8 chunks][128 rows][8]): K step
// kk covers chunks 2kk and 2kk + 1.
__device__ __forceinline__ uint64_t rows_kmajor_desc(uint32_t addr, int kk) {
  return smem_desc(addr + (uint32_t)kk * 2u * kMqRows * 16u, kMqRows * 16, 128, kSwizzleNone);
}
// B operand K tile (64 keys x 128 d, K-major, two 128-byte-swizzled boxes of 64 d).
__device__ __forceinline__ uint64_t ktile_kmajor_desc(uint32_t tile, int kk) {
  const uint32_t start = tile + (uint32_t)(kk >> 2) * kMqBox + (uint32_t)(kk & 3) * 32u;
  return smem_desc(start, 16, 1024, kSwizzle128B);
}
// B operand V tile (N = 128 d, K = 64 keys, MN-major, two swizzled boxes of 64 d):
// K step kk covers keys [16kk, 16kk + 16).
__device__ __forceinline__ uint64_t vtile_mnmajor_desc(uint32_t tile, int kk) {
  return smem_desc(tile + (uint32_t)kk * 16u * 128u, kMqBox, 1024, kSwizzle128B);
}

}  // namespace

template <int H>
__global__ void __launch_bounds__(kMqThreads, 1)
    full_attn_mq_kernel(const __grid_constant__ CUtensorMap tmap_k,
                        const __grid_constant__ CUtensorMap tmap_v, FullParams p, int n_groups) {
  using L = MqSmem;
  constexpr int NS = L::kStages;
  constexpr int G = kMqRows / H;  // tokens per CTA
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* kst = smem + L::kKOff;
  uint8_t* vst = smem + L::kVOff;
  uint8_t* qs = smem + L::kQOff;
  uint8_t* ps = smem + L::kPOff;
  float* red = reinterpret_cast<float*>(smem + L::kRedOff);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* kfull = bars;
  uint64_t* kempty = bars + NS;
  uint64_t* vfull = bars + 2 * NS;
  uint64_t* vempty = bars + 3 * NS;
  uint64_t* s_full = bars + 4 * NS;  // [2]
  uint64_t* s_free = s_full + 2;     // [2]
  uint64_t* p_full = s_full + 4;     // [2]
  uint64_t* p_free = s_full + 6;     // [2]
  uint64_t* mma_done = s_full + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kSlotOff);

  const int warp = threadIdx.x >> 5;
  const int split = blockIdx.x;
  const int grp = blockIdx.y % n_groups, b = blockIdx.y / n_groups;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(kfull + s, 1);
      mbar_init(kempty + s, 1);
      mbar_init(vfull + s, 1);
      mbar_init(vempty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(s_full + s, 1);
      mbar_init(s_free + s, kMqSoftmax);
      mbar_init(p_full + s, kMqSoftmax);
      mbar_init(p_free + s, 1);
    }
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane_id() == 0) {
    prefetch_tmap(&tmap_k);
    prefetch_tmap(&tmap_v);
  }
  griddep_wait();

  const int t0 = grp * G;                       // first token of the group
  const int ntok = min(G, p.n_q - t0);
  const int Lb = seq_len(p.kv, b, p.n_q, p.status, split == 0 && grp == 0);
  const int pos0 = Lb - p.n_q + t0;             // position of the group's first token
  const int k0 = split * p.chunk1;
  const int k1 = min(k0 + p.chunk1, pos0 + ntok);  // the group's last token sees [0, k1)
  const int n_tiles = k0 < k1 ? (k1 - k0 + kMqKeys - 1) / kMqKeys : 0;
  auto part_index = [&](int g) {  // partial slot of token t0 + g for this split
    return ((size_t)b * p.n_q + t0 + g) * p.splits1 + split;
  };
  bool ok = true;

  if (n_tiles == 0) {
    for (int r = threadIdx.x; r < ntok * H; r += blockDim.x) {
      const size_t pi = part_index(r / H) * H + r % H;
      p.part_ml[pi * 2] = -INFINITY;
      p.part_ml[pi * 2 + 1] = 0.f;
    }
  } else {
    // Q rows (token g, head h) at row g * H + h; rows of absent tokens are zero.
    for (int e = threadIdx.x; e < kMqRows * (kHeadDim / 8); e += blockDim.x) {
      const int r = e % kMqRows, c = e / kMqRows;
      const int g = r / H, h = r % H;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (g < ntok)
        v = *reinterpret_cast<const uint4*>(
            p.q + (((size_t)b * p.n_q + t0 + g) * H + h) * kHeadDim + c * 8);
      *reinterpret_cast<uint4*>(qs + c * (kMqRows * 16) + r * 16) = v;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const uint32_t tmem_o = tmem_base + 2 * kMqKeys;

    if (warp == 0) {
      // ------------------------------------------------------------ TMA producer
      if (elect_one()) {
        const uint64_t pol = policy_evict_last();  // the other groups read the same tiles
        const int row0 = b * p.kv.max_len + k0;
        int issued = 0;
        for (int i = 0; i < n_tiles && ok; ++i) {
          const int s = i % NS;
          const uint32_t ph = ((i / NS) & 1) ^ 1;
          const int row = row0 + i * kMqKeys;
          if (!mbar_wait(kempty + s, ph)) { ok = false; break; }
          mbar_arrive_expect_tx(kfull + s, kMqTile);
          tma_load_2d(kst + s * kMqTile, &tmap_k, kfull + s, 0, row, pol);
          tma_load_2d(kst + s * kMqTile + kMqBox, &tmap_k, kfull + s, 64, row, pol);
          if (!mbar_wait(vempty + s, ph)) { ok = false; break; }
          mbar_arrive_expect_tx(vfull + s, kMqTile);
          tma_load_2d(vst + s * kMqTile, &tmap_v, vfull + s, 0, row, pol);
          tma_load_2d(vst + s * kMqTile + kMqBox, &tmap_v, vfull + s, 64, row, pol);
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
        const uint32_t id_qk = idesc_f16(kMqRows, kMqKeys, true, false, false);
        const uint32_t id_pv = idesc_f16(kMqRows, kHeadDim, true, false, true);
        const uint32_t q_addr = smem_u32(qs);
        auto issue_pv = [&](int t) -> bool {
          const int s = t % NS, pb = t & 1;
          if (!mbar_wait(vfull + s, (t / NS) & 1)) return false;
          if (!mbar_wait(p_full + pb, (t >> 1) & 1)) return false;
          tc_fence_after();
          const uint32_t v_addr = smem_u32(vst + s * kMqTile);
          const uint32_t p_hi = smem_u32(ps + (2 * pb) * L::kPBytes);
          const uint32_t p_lo = p_hi + L::kPBytes;
#pragma unroll
          for (int kk = 0; kk < kMqKeys / 16; ++kk)
            mma_f16_ss(tmem_o, rows_kmajor_desc(p_hi, kk), vtile_mnmajor_desc(v_addr, kk), id_pv,
                       (t > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < kMqKeys / 16; ++kk)
            mma_f16_ss(tmem_o, rows_kmajor_desc(p_lo, kk), vtile_mnmajor_desc(v_addr, kk), id_pv,
                       1u);
          mma_commit(p_free + pb);
          mma_commit(vempty + s);
          return true;
        };
        for (int i = 0; i < n_tiles && ok; ++i) {
          const int s = i % NS, sb = i & 1;
          if (!mbar_wait(kfull + s, (i / NS) & 1)) { ok = false; break; }
          if (!mbar_wait(s_free + sb, ((i >> 1) & 1) ^ 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t k_addr = smem_u32(kst + s * kMqTile);
#pragma unroll
          for (int kk = 0; kk < kHeadDim / 16; ++kk)
            mma_f16_ss(tmem_base + sb * kMqKeys, rows_kmajor_desc(q_addr, kk),
                       ktile_kmajor_desc(k_addr, kk), id_qk, kk > 0 ? 1u : 0u);
          mma_commit(s_full + sb);
          mma_commit(kempty + s);
          if (i > 0 && !issue_pv(i - 1)) { ok = false; break; }
        }
        if (ok && !issue_pv(n_tiles - 1)) ok = false;
        mma_commit(mma_done);
        if (!mbar_wait(mma_done, 0)) ok = false;
      }
    } else {
      // ------------------------------------------------------------ softmax
      const int lg = warp & 3;                 // TMEM lane quarter of this warp
      const int half = (warp - 2) >> 2;        // which 32 keys of a tile (and half of O)
      const int r = lg * 32 + (int)lane_id();  // query row == TMEM lane
      const int st = half * kMqRows + r;       // softmax thread index, 0 .. 255
      const uint32_t lane_base = (uint32_t)(lg * 32) << 16;
      const int g = r / H;
      const bool row_live = g < ntok;
      const int pos_r = pos0 + g;                // this row's token sees keys [0, pos_r]
      const int kend = row_live ? min(k1, pos_r + 1) : k0;  // its keys in this chunk
      const float c2 = p.sm_scale * kLog2eMq;
      constexpr int KH = kMqKeys / 2;            // keys per thread per tile
      float mref = -INFINITY, l = 0.f;
      for (int i = 0; i < n_tiles; ++i) {
        const int sb = i & 1;
        if (ok && !mbar_wait(s_full + sb, (i >> 1) & 1)) ok = false;
        if (named_bar_or(3, kMqSoftmax, !ok)) ok = false;
        tc_fence_after();
        float x[KH];  // raw logits s (the log2-domain value is s * c2)
        {
          uint32_t v[KH];
#pragma unroll
          for (int c = 0; c < KH; c += 16)
            tmem_ld16(tmem_base + lane_base + sb * kMqKeys + half * KH + c,
                      *reinterpret_cast<uint32_t(*)[16]>(v + c));
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < KH; ++e) x[e] = __uint_as_float(v[e]);
        }
        tc_fence_before();
        mbar_arrive(s_free + sb);
        const int jb = k0 + i * kMqKeys + half * KH;
        if (jb + KH > kend) {  // only tiles at the chunk end or the causal edge are masked
#pragma unroll
          for (int c = 0; c < KH; ++c)
            if (jb + c >= kend) x[c] = -INFINITY;
        }
        float tmax = -INFINITY;
#pragma unroll
        for (int c = 0; c < KH; ++c) tmax = fmaxf(tmax, x[c]);
        tmax *= c2;  // c2 > 0: the max of the scaled logits
        // Row max over both halves (slots alternate by tile so that a fast thread
        // cannot overwrite a value its partner has not read yet).
        float* rt = red + (size_t)(i & 1) * 2 * kMqRows;
        rt[half * kMqRows + r] = tmax;
        named_bar_sync(1, kMqSoftmax);
        tmax = fmaxf(rt[r], rt[kMqRows + r]);
        // Lazy reference: move it only when this tile would give p > 2^8.
        const bool move = tmax - mref > kRescaleAtMq;  // false while tmax is -inf
        float alpha = 1.f;
        if (move) {
          alpha = exp2f(mref - tmax);  // 0 while mref is -inf
          mref = tmax;
          l *= alpha;
        }
        if (__any_sync(0xffffffffu, move) && i > 0) {
          // O holds the P.V of tiles < i: wait for the last one, then rescale this
          // thread's half of the row (rows whose reference stayed multiply by 1).
          if (ok && !mbar_wait(p_free + ((i - 1) & 1), ((i - 1) >> 1) & 1)) ok = false;
          tc_fence_after();
          uint32_t v[64];
#pragma unroll
          for (int c = 0; c < 64; c += 16)
            tmem_ld16(tmem_o + lane_base + half * 64 + c, *reinterpret_cast<uint32_t(*)[16]>(v + c));
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 64; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
#pragma unroll
          for (int c = 0; c < 64; c += 16)
            tmem_st16(tmem_o + lane_base + half * 64 + c,
                      *reinterpret_cast<const uint32_t(*)[16]>(v + c));
          tmem_wait_st();
          tc_fence_before();
        }
        // P for this tile into buffer sb (free once the P.V of tile i-2 is done).
        if (ok && i >= 2 && !mbar_wait(p_free + sb, ((i >> 1) & 1) ^ 1)) ok = false;
        uint8_t* phi = ps + (2 * sb) * L::kPBytes;
        uint8_t* plo = phi + L::kPBytes;
        const float nmr = -finite_ref(mref);
#pragma unroll
        for (int c = 0; c < KH / 8; ++c) {
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float p0 = ex2_ftz(fmaf(x[c * 8 + 2 * e], c2, nmr));
            const float p1 = ex2_ftz(fmaf(x[c * 8 + 2 * e + 1], c2, nmr));
            l += p0 + p1;
            split_bf16_hi_lo(p0, p1, hw[e], lw[e]);
          }
          const int chunk = half * (KH / 8) + c;  // 8-key chunk of the tile
          *reinterpret_cast<uint4*>(phi + chunk * (kMqRows * 16) + r * 16) =
              make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(plo + chunk * (kMqRows * 16) + r * 16) =
              make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
        if (i == n_tiles - 1 && half == 0 && r < kMqKeys && k0 + i * kMqKeys + r >= k1) {
          // Rows past the chunk end may hold anything (NaN included); 0 * NaN would
          // poison P.V, so zero this key's V row once its tile has landed.
          const int s = i % NS;
          if (ok && !mbar_wait(vfull + s, (i / NS) & 1)) ok = false;
          uint4* v0 = reinterpret_cast<uint4*>(vst + s * kMqTile + r * 128);
          uint4* v1 = reinterpret_cast<uint4*>(vst + s * kMqTile + kMqBox + r * 128);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            v0[e] = make_uint4(0, 0, 0, 0);
            v1[e] = make_uint4(0, 0, 0, 0);
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(p_full + sb);
      }
      griddep_launch_dependents();  // the merge may be scheduled; it waits for this grid
      // Epilogue: row r of O is (token g, head h); each thread writes its half of the
      // row, the half-0 thread the row's (m, l) with l summed over both halves.
      const int last = n_tiles - 1;
      if (ok && !mbar_wait(p_free + (last & 1), (last >> 1) & 1)) ok = false;
      tc_fence_after();
      const size_t pi = part_index(row_live ? g : 0) * H + r % H;
      float* po = p.part_o + pi * kHeadDim + half * 64;
      {
        uint32_t v[64];
#pragma unroll
        for (int c = 0; c < 64; c += 16)
          tmem_ld16(tmem_o + lane_base + half * 64 + c, *reinterpret_cast<uint32_t(*)[16]>(v + c));
        tmem_wait_ld();
        if (row_live) {
#pragma unroll
          for (int e = 0; e < 64; e += 4)
            *reinterpret_cast<float4*>(po + e) =
                make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                            __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
        }
      }
      tc_fence_before();
      named_bar_sync(1, kMqSoftmax);  // every thread is past its last use of red
      red[st] = l;
      named_bar_sync(1, kMqSoftmax);
      if (row_live && half == 0) {
        p.part_ml[pi * 2] = mref;
        p.part_ml[pi * 2 + 1] = red[r] + red[kMqRows + r];
      }
    }
  }
  if (!ok) set_status(p.status, HS2_ERR_DEVICE_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(*tmem_slot, L::kTmemCols);
  }
}

template <int H>
static cudaError_t launch_mq_t(const FullParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                               int batch, int n_groups, cudaStream_t st) {
  using L = MqSmem;
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(full_attn_mq_kernel<H>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::kBytes);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  return launch_pdl(full_attn_mq_kernel<H>, dim3(p.splits1, batch * n_groups),
                    dim3(kMqThreads), L::kBytes, st, tk, tv, p, n_groups);
}

int mq_tokens_per_cta(int h) { return h >= 16 && h <= kMqRows ? kMqRows / h : 0; }

cudaError_t launch_full_attn_mq(const FullParams& p, const CUtensorMap& tk, const CUtensorMap& tv,
                                int batch, cudaStream_t st) {
  const int G = mq_tokens_per_cta(p.h);
  if (G < 1) return cudaErrorInvalidValue;
  const int n_groups = (p.n_q + G - 1) / G;
  switch (p.h) {
    case 16: return launch_mq_t<16>(p, tk, tv, batch, n_groups, st);
    case 32: return launch_mq_t<32>(p, tk, tv, batch, n_groups, st);
    case 48: return launch_mq_t<48>(p, tk, tv, batch, n_groups, st);
    case 64: return launch_mq_t<64>(p, tk, tv, batch, n_groups, st);
    case 128: return launch_mq_t<128>(p, tk, tv, batch, n_groups, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace hs2
