// Self-test of the kernels' bounded wait (sm_100a): one warp waits on an mbarrier phase
// that nothing completes, through the same mbar_wait the decode kernels use, with a
// short limit.  The wait must run out, set PA_DEVERR_TIMEOUT in the device error flag
// and return, leaving the context usable; no load or copy is in flight.

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

__global__ void selftest_wait_kernel(int32_t* err, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&bar), 1);  // one arrival completes phase 0; none comes
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  mbar_wait(smem_addr(&bar), 0, threadIdx.x == 0 ? err : nullptr, limit_ns);
}

}  // namespace
}  // namespace pa

extern "C" pa_status pa_selftest_bounded_wait(int32_t* dev_err_flag, unsigned limit_us,
                                              pa_stream_t stream) {
  if (!dev_err_flag || limit_us == 0 || limit_us > 1000000u) return PA_ERR_INVALID_ARG;
  pa::selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      dev_err_flag, static_cast<uint64_t>(limit_us) * 1000ull);
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
