// hs2_sparse_attn_noalloc: the reusing sparse-attention layer without a caller
// workspace.
//
// Some callers cannot allocate device memory when they call this layer: a serving
// runtime that hands out all device memory from its own pre-planned pool and forbids
// stray allocations, a plugin loaded into a host framework that owns the allocator,
// or a plain C caller that keeps no buffer alive between calls.  cudaMalloc may also
// synchronise the device, which such callers cannot afford in the middle of a step.
// For them this entry point keeps the layer's scratch (the split partials) in a fixed
// array that lives in the library's own device memory:
// every GPU that loads the library holds kNoAllocScratchBytes of it until the
// process exits.  The caller still passes the inputs and the output.
//
// The array is shared by every call on a device and keeps what the last call left in
// it; every call rewrites all the partials it reads, so nothing needs clearing.  Two
// calls whose kernels overlap on the GPU (different streams without ordering between
// them) race on the array and give wrong results: serialise them.
#include <mutex>

#include "hs2_internal.cuh"

namespace hs2 {
namespace {

constexpr size_t kNoAllocScratchBytes = 4u << 20;  // 4 MiB per device
constexpr int kNoAllocMaxDevices = 64;
constexpr int kChunkRows = 64;                     // index entries per CTA, as hs2_sparse_attn

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kNoAllocMaxDevices] = {};

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// Device address of the scratch array on the current device, resolved once per device.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace hs2

using namespace hs2;

extern "C" HS2_API hs2_status hs2_sparse_attn_noalloc(const void* q_layer, int n_q, int h_q,
                                                     const hs2_kv* kv, const int32_t* idx,
                                                     int idx_width, float sm_scale, float* out,
                                                     uint32_t* device_status,
                                                     hs2_stream_t stream) {
  if (!kv || !kv->k || !kv->v || !kv->lens || !q_layer || !idx || !out)
    return HS2_ERR_INVALID_ARGUMENT;
  if (kv->head_dim != kHeadDim) return HS2_ERR_UNSUPPORTED;
  const bool fp8 = kv->dtype == HS2_KV_FP8_E4M3;
  if (kv->dtype != HS2_KV_BF16 && !fp8) return HS2_ERR_UNSUPPORTED;
  if (fp8 != (kv->k_scale != nullptr) || fp8 != (kv->v_scale != nullptr))
    return HS2_ERR_INVALID_ARGUMENT;
  if (kv->batch < 1 || kv->max_len < 1 || n_q > kv->max_len) return HS2_ERR_INVALID_ARGUMENT;
  if (n_q < 1 || n_q > kMaxNq || h_q < 16 || h_q > kMaxHeads || (h_q % 16) != 0)
    return HS2_ERR_UNSUPPORTED;
  if (idx_width < 1 || idx_width > kMaxIdxWidth) return HS2_ERR_UNSUPPORTED;
  if ((long long)kv->batch * kv->max_len >= (1ll << 31)) return HS2_ERR_UNSUPPORTED;
  const uintptr_t align = (uintptr_t)q_layer | (uintptr_t)out | (uintptr_t)kv->k |
                          (uintptr_t)kv->v;
  if (align & 15u) return HS2_ERR_INVALID_ARGUMENT;

  // Scratch layout: [status word][partial o][partial (m, l)].
  const size_t bq = (size_t)kv->batch * n_q;
  const int splits = (idx_width + kChunkRows - 1) / kChunkRows;
  const size_t off_o = 256;
  const size_t off_ml = off_o + round256(bq * splits * h_q * kHeadDim * sizeof(float));
  const size_t need = off_ml + round256(bq * splits * h_q * 2 * sizeof(float));
  if (need > kNoAllocScratchBytes) return HS2_ERR_WORKSPACE_TOO_SMALL;

  void* base = nullptr;
  cudaError_t e = scratch_address(&base);
  if (e != cudaSuccess) return HS2_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;

  SparseParams p;
  p.q = static_cast<const uint16_t*>(q_layer);
  p.kv.k = kv->k;
  p.kv.v = kv->v;
  p.kv.k_scale = kv->k_scale;
  p.kv.v_scale = kv->v_scale;
  p.kv.lens = kv->lens;
  p.kv.batch = kv->batch;
  p.kv.max_len = kv->max_len;
  p.kv.fp8 = fp8;
  p.idx = idx;
  p.n_q = n_q;
  p.h = h_q;
  p.idx_width = idx_width;
  p.sm_scale = sm_scale;
  p.splits4 = splits;
  p.chunk4 = kChunkRows;
  p.part_o = reinterpret_cast<float*>(static_cast<char*>(base) + off_o);
  p.part_ml = reinterpret_cast<float*>(static_cast<char*>(base) + off_ml);
  p.status = device_status ? device_status : static_cast<uint32_t*>(base);
  e = launch_sparse_attn(p, kv->batch, s);
  if (e != cudaSuccess) return HS2_ERR_CUDA;
  MergeParams m;
  m.part_o = p.part_o;
  m.part_ml = p.part_ml;
  m.splits = splits;
  m.h = h_q;
  m.out = out;
  m.lse_out = nullptr;
  m.lse64 = nullptr;
  e = launch_merge(m, (int)bq, false, s);
  return e == cudaSuccess ? HS2_OK : HS2_ERR_CUDA;
}
