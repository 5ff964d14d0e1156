// noalloc.cu -- spkv_decode_attention_static_ws: ADA decode attention whose
// split-partials workspace lives in this library's own device memory, so the
// caller passes no workspace and nothing is allocated at call time.
//
// Who needs it: callers that cannot call cudaMalloc (or any allocator) when
// they decode -- for example a serving loop that runs under a fixed memory
// budget checked at start-up, a runtime whose allocator is not reachable from
// the thread that issues the decode, or a host program that must not touch
// the CUDA allocator after initialisation.  They give up the freedom to size
// the workspace: it is a fixed array, and every call shares it.
#include <cuda_runtime.h>

#include <mutex>

#include "spkv.h"

namespace {

// The scratch array: one per device that loads the library, held until the
// process exits.  In host code this name is only a stand-in for the device
// symbol; the kernels get its device address from cudaGetSymbolAddress.
constexpr size_t kStaticWsBytes = SPKV_STATIC_WS_BYTES;
static __device__ __align__(256) unsigned char g_static_ws[kStaticWsBytes];

std::mutex g_mu;
void *g_ws_addr[64];  // device address of g_static_ws, per device ordinal

// Device address of the array on the current device, looked up once per
// device (with that device current) and cached.
cudaError_t static_ws_address(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_ws_addr[dev]) {
    void *ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_static_ws);
    if (e != cudaSuccess) return e;
    g_ws_addr[dev] = ptr;
  }
  *out = g_ws_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" spkv_status spkv_decode_attention_static_ws(const spkv_cache *cache, const uint16_t *q, int32_t B,
                                                       int32_t num_q_heads, const int32_t *block_table,
                                                       int32_t max_pages, const int32_t *ctx_lens, int32_t max_ctx,
                                                       void *out, int32_t out_is_bf16, int32_t num_splits,
                                                       void *stream) {
  if (!cache || cache->num_kv_heads < 1) return SPKV_ERR_INVALID_ARG;
  if (B < 0 || num_q_heads < 1 || max_ctx < 0 || num_splits < 0) return SPKV_ERR_INVALID_ARG;
  if (B == 0) return SPKV_OK;
  const size_t need = spkv_decode_workspace_bytes(B, num_q_heads, cache->num_kv_heads, max_ctx, num_splits);
  if (need == 0) return SPKV_ERR_INVALID_ARG;
  if (need > kStaticWsBytes) return SPKV_ERR_WORKSPACE;  // beyond the fixed array
  void *ws = nullptr;
  if (static_ws_address(&ws) != cudaSuccess) return SPKV_ERR_CUDA;
  // Every partial the merge reads is written by the same call first: nothing
  // in the array has to start at zero.
  return spkv_decode_attention(cache, q, B, num_q_heads, block_table, max_pages, ctx_lens, max_ctx, out,
                               out_is_bf16, ws, kStaticWsBytes, num_splits, stream);
}
