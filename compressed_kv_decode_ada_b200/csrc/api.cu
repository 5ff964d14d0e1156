// api.cu -- status strings and per-device properties for libspkv.
#include <cuda.h>
#include <cuda_runtime.h>

#include "spkv.h"

namespace spkv {

// Tensor map of a bf16 value-page array [num_pages, H_kv, 16, 128] seen as a
// 3-D tensor (64 columns of a half row, token row, half) whose box {64, 16, 2}
// is one whole page, with the 128-byte shared-memory swizzle.  The encoder is
// obtained from the driver through the runtime (no link against libcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool make_value_tensor_map(CUtensorMap *map, const void *v_pages, uint64_t rows) {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !f)
      return false;
    fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  if (rows == 0 || rows > 0xffffffffull) return false;
  // (dim 64 within a half row, token row, half): one box {64, 16, 2} is a
  // whole 16 x 128 page, landing as [half][token][64] so that each 128-byte
  // line of the 128-byte swizzle is (half, token)
  const cuuint64_t dims[3] = {64, rows, 2};
  const cuuint64_t strides[2] = {256, 128};
  const cuuint32_t box[3] = {64, 16, 2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(v_pages), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

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
