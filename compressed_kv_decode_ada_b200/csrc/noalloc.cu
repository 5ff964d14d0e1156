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
#include <cuda.h>
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
void *g_ws_addr[64];                // device address of g_static_ws, per device ordinal
unsigned long long g_ws_ctx[64];    // id of the context that address belongs to

// Driver entry points for the current context and its id (a 64-bit value
// unique over the process's lifetime, so a context destroyed and created
// again -- cudaDeviceReset, a released primary context -- gets a new id even
// when it reuses the old handle).
typedef CUresult (*ctx_get_current_fn)(CUcontext *);
typedef CUresult (*ctx_get_id_fn)(CUcontext, unsigned long long *);
ctx_get_current_fn g_get_current = nullptr;
ctx_get_id_fn g_get_id = nullptr;
bool g_entry_tried = false;

// Id of the context current on this thread; 0 when there is none yet or the
// driver does not give one.  Called with g_mu held.
unsigned long long current_ctx_id() {
  if (!g_entry_tried) {
    g_entry_tried = true;
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_get_current = reinterpret_cast<ctx_get_current_fn>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_get_id = reinterpret_cast<ctx_get_id_fn>(f);
  }
  if (!g_get_current || !g_get_id) return 0;
  CUcontext ctx = nullptr;
  if (g_get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  unsigned long long id = 0;
  if (g_get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of the array in the current context.  It is looked up
// (cudaGetSymbolAddress, with the device current) on the first call in a
// context and cached with the context's id; a call from another context of
// the device -- after a device reset, say, when the module has been loaded
// again at another address -- looks it up again.
cudaError_t static_ws_address(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  const unsigned long long id = current_ctx_id();
  if (!g_ws_addr[dev] || id == 0 || id != g_ws_ctx[dev]) {
    void *ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_static_ws);  // makes the device's primary context current if none is
    if (e != cudaSuccess) return e;
    g_ws_addr[dev] = ptr;
    g_ws_ctx[dev] = id ? id : current_ctx_id();
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
  // spkv_decode_attention's own argument checks come first: given no
  // workspace it launches nothing and returns SPKV_ERR_WORKSPACE exactly when
  // every other argument is valid (SPKV_OK when B = 0), so a bad argument
  // gets the status it gets there.
  const spkv_status chk = spkv_decode_attention(cache, q, B, num_q_heads, block_table, max_pages, ctx_lens, max_ctx,
                                                out, out_is_bf16, nullptr, 0, num_splits, stream);
  if (chk != SPKV_ERR_WORKSPACE) return chk;
  if (B == 0) return SPKV_OK;  // nothing to do
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
