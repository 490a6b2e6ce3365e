// attn_decode_fixedsplit_noalloc: the fixed-split decode attention for callers
// that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc or hand the library a workspace: code
// embedded in a host application whose device-memory budget is owned and
// fully pre-committed by someone else, plug-ins that get no allocator handle,
// and latency-critical paths where an allocation (which may synchronise the
// device) is not allowed.  For them this entry point keeps the attention's
// split partials in a file-scope device array instead of a caller workspace.
//
// The array is kNoallocScratchBytes (34 MiB) and lives on every GPU that
// loads the library until the process exits.  Its device address is looked up
// once per device, with that device current, on the first call on that
// device; make that first call before any stream capture.  Every call on a
// device shares the one array and leaves the last call's partials in it:
// calls whose kernels overlap on the GPU (different streams, no ordering)
// race on it.  Nothing in it needs clearing between calls -- the split kernel
// writes every partial the combine kernel reads.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace {

constexpr size_t kNoallocScratchBytes = size_t(34) << 20;

static __device__ __align__(256) unsigned char g_attn_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of g_attn_scratch on the current device (host code may not
// use the symbol itself: on the host it is only a stand-in).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return INV_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_attn_scratch) != cudaSuccess || p == nullptr) return INV_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return INV_OK;
}

}  // namespace

extern "C" int attn_decode_fixedsplit_noalloc(const float* q, int B, int n_heads, const inv_kv_cache* cache,
                                              const int32_t* slot, const int32_t* len, int max_len_bound, int split,
                                              float softmax_scale, float* out, uint16_t* out_hi, uint16_t* out_lo,
                                              inv_stream stream) {
  if (!cache || B < 0 || n_heads <= 0) return INV_ERR_INVALID_ARG;
  if (split != INV_KV_SPLIT) return INV_ERR_UNSUPPORTED_SHAPE;
  if (cache->head_dim != INV_HEAD_DIM || cache->n_kv_heads <= 0 || n_heads % cache->n_kv_heads != 0)
    return INV_ERR_UNSUPPORTED_SHAPE;
  const int G = n_heads / cache->n_kv_heads;
  if (G != 1 && G != 2 && G != 4) return INV_ERR_UNSUPPORTED_SHAPE;
  if (cache->max_len <= 0 || cache->max_len % 64 != 0 || cache->n_slots <= 0) return INV_ERR_INVALID_ARG;
  if ((uint64_t)cache->n_slots * cache->n_kv_heads * cache->max_len >= (1ull << 31)) return INV_ERR_UNSUPPORTED_SHAPE;
  if (B == 0) return INV_OK;
  if (B > 65535) return INV_ERR_UNSUPPORTED_SHAPE;
  if (!q || !slot || !len || !out || !cache->k || !cache->v || !cache->k_scale || !cache->v_scale)
    return INV_ERR_INVALID_ARG;
  if ((out_hi == nullptr) != (out_lo == nullptr)) return INV_ERR_INVALID_ARG;
  if (!inv::aligned16(q) || !inv::aligned16(cache->k) || !inv::aligned16(cache->v) || !inv::aligned16(out))
    return INV_ERR_INVALID_ARG;
  if (out_hi && ((reinterpret_cast<uintptr_t>(out_hi) | reinterpret_cast<uintptr_t>(out_lo)) & 7u))
    return INV_ERR_INVALID_ARG;
  const int mlb =
      max_len_bound > 0 ? (max_len_bound < cache->max_len ? max_len_bound : cache->max_len) : cache->max_len;
  if (inv::attn_workspace_bytes(B, n_heads, mlb) > kNoallocScratchBytes) return INV_ERR_WORKSPACE;
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != INV_OK) return rc;
  return inv::launch_attention(q, B, n_heads, *cache, slot, len, mlb, softmax_scale, out, out_hi, out_lo, scratch,
                               static_cast<cudaStream_t>(stream), -1);
}
