// selftest.cu -- failure detection without a fault: a bounded wait that runs
// out on purpose.
//
// Every spin-wait in this library gives up after a time limit, latches
// kErrTimeout in the device's error word and returns, so a lost signal ends
// as an error status from sbl_check instead of a hung device.  This kernel
// takes that path deliberately: one thread waits on an mbarrier phase that
// nothing completes (no thread ever arrives), with the library's try-wait /
// global-timer pattern, until the caller's limit passes.  It then latches
// the timeout and exits; the CUDA context stays usable.
#include <cuda_runtime.h>
#include <cstdint>

#include "sbl_device.cuh"
#include "sbl_internal.h"

namespace sbl {
namespace {

__global__ void wait_timeout_selftest_kernel(uint64_t limit_ns, uint32_t* err) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_mbar_init();
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(&bar, 0)) {  // phase 0 needs one arrival, and none comes
    if (globaltimer_ns() - t0 > limit_ns) {
      latch_error(err, kErrTimeout);
      return;
    }
    __nanosleep(1000);
  }
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(uint64_t limit_ns, cudaStream_t stream, uint32_t* err) {
  wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(limit_ns, err);
  return cudaGetLastError();
}

}  // namespace sbl
