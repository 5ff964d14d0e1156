// api.cu -- status strings and per-device properties for libspkv.
#include <cuda_runtime.h>

#include "spkv.h"

namespace spkv {

// Streaming-multiprocessor count of the current device (cached per device).
int device_sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
  if (cached[dev] <= 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    cached[dev] = n;
  }
  return cached[dev];
}

}  // namespace spkv

extern "C" const char *spkv_status_string(spkv_status s) {
  switch (s) {
    case SPKV_OK: return "SPKV_OK";
    case SPKV_ERR_INVALID_ARG: return "SPKV_ERR_INVALID_ARG";
    case SPKV_ERR_UNSUPPORTED: return "SPKV_ERR_UNSUPPORTED";
    case SPKV_ERR_WORKSPACE: return "SPKV_ERR_WORKSPACE";
    case SPKV_ERR_CUDA: return "SPKV_ERR_CUDA";
  }
  return "SPKV_ERR_UNKNOWN";
}
