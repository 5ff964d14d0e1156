// debug.cu -- spkv_debug_wait_timeout: a test hook for the bounded waits.
//
// Every wait of the decode kernels on an mbarrier gives up after a time limit
// (about 1 s), sets SPKV_DEVERR_TIMEOUT and lets the kernel run out without
// waiting, so a lost copy or a stuck warp ends as a readable error instead of
// a hung GPU.  This hook runs that same wait routine on an mbarrier that
// nothing ever completes, with a short limit, so a test can see it give up,
// set the flag and return.
#include "spkv_common.cuh"

namespace spkv {
namespace {

__global__ void __launch_bounds__(32) wait_timeout_kernel(uint32_t *err, int32_t *status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // one arrival expected; none ever comes
    abort_flag = 0;
    mbar_fence_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    const uint64_t t0 = globaltimer_ns();
    const bool ok = mbar_wait_bounded(&bar, 0u, &abort_flag, err, 0u, limit_ns);
    status[0] = ok ? 0 : 1;  // 1: the wait gave up
    status[1] = (int32_t)((globaltimer_ns() - t0) / 1000u);  // microseconds waited
    status[2] = abort_flag;
  }
}

}  // namespace
}  // namespace spkv

extern "C" spkv_status spkv_debug_wait_timeout(uint32_t *err_flags, int32_t *status, uint64_t limit_ns,
                                               void *stream) {
  using namespace spkv;
  if (!err_flags || !status || limit_ns == 0 || limit_ns > 1000000000ull) return SPKV_ERR_INVALID_ARG;
  wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(err_flags, status, limit_ns);
  return cudaGetLastError() == cudaSuccess ? SPKV_OK : SPKV_ERR_CUDA;
}
