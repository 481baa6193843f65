// pa_selftest_wait_timeout: makes one pipeline wait run out on purpose, so
// that the time-limited wait every kernel of the library uses can be tested
// without hanging or faulting anything.
//
// One CTA of two warps.  Warp 1 allocates tensor memory the way the prefill
// kernel's MMA warp does; warp 0 waits, warp-uniformly, on an mbarrier phase
// that nothing completes, exactly as a softmax warp waits for its scores.
// The wait gives up after the caller's limit and records code 1 in the
// device error word; the CTA then takes the same exit path as the kernels
// (tcgen05 fences around a CTA barrier, tensor memory freed) and returns.
#include <cuda_runtime.h>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

constexpr uint32_t kSelftestTmemCols = 32;

__global__ void __launch_bounds__(64, 1) wait_timeout_kernel(unsigned int* err, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t tmem_slot;
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);   // one arrival completes the phase; none ever comes
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, kSelftestTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) mbar_wait_warp(&bar, 0, err, limit_ns);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_slot, kSelftestTmemCols);
}

}  // namespace
}  // namespace pa

extern "C" pa_status pa_selftest_wait_timeout(int64_t limit_ns, void* stream) {
  if (limit_ns < 1000 || limit_ns > 1000000000) {
    pa::set_last_error("selftest_wait_timeout: limit_ns must lie in [1e3, 1e9]");
    return PA_ERR_INVALID_ARG;
  }
  pa::set_last_error("%s", "");
  pa::wait_timeout_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(
      pa::current_device_info()->error_word, static_cast<uint64_t>(limit_ns));
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    pa::set_last_error("selftest_wait_timeout launch: %s", cudaGetErrorString(e));
    return PA_ERR_CUDA;
  }
  return PA_OK;
}
