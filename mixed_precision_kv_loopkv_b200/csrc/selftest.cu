// Self-test of the kernels' bounded waits (sm_100a).
//
// Every wait of the LoopKV kernels on an mbarrier gives up after a fixed time
// (kWaitTimeoutNs, read from the global timer), reports
// LOOPKV_DEVERR_TIMEOUT and lets the CTA finish, so that a copy that never
// lands cannot hang the device.  This entry point runs that wait on a
// barrier whose phase can never complete (one arrival announcing 16 bytes
// that no copy delivers) and reports what the wait did.
#include <stdint.h>

#include "device_common.cuh"
#include "loopkv.h"

namespace loopkv {
namespace {

__global__ void wait_timeout_kernel(int32_t* err, unsigned long long* elapsed_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_addr(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    fence_mbar_init();
    // the arrival is counted, the 16 bytes never are: the phase stays open
    mbar_arrive_expect_tx(b, 16);
    const unsigned long long t0 = global_timer_ns();
    const bool done = mbar_wait(b, 0);
    *elapsed_ns = global_timer_ns() - t0;
    if (!done) flag_error(err, LOOPKV_DEVERR_TIMEOUT);
  }
}

}  // namespace
}  // namespace loopkv

extern "C" {

loopkv_status loopkv_selftest_wait_timeout(int32_t* err_flag, uint64_t* elapsed_ns, void* stream) {
  if (!err_flag || !elapsed_ns) return LOOPKV_ERR_INVALID_ARG;
  loopkv::wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      err_flag, reinterpret_cast<unsigned long long*>(elapsed_ns));
  return cudaGetLastError() == cudaSuccess ? LOOPKV_OK : LOOPKV_ERR_CUDA;
}

}  // extern "C"
