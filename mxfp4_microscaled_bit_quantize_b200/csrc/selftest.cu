// Self-test of the library's failure detection: a kernel whose mbarrier phase never completes.
// Warp 0 waits with the same bounded wait every pipeline kernel uses (mbar_wait: hardware
// suspend between polls, %globaltimer bound); when the bound runs out it records its code in the
// status word and raises the CTA abort flag. Warp 1 waits on the same phase and must leave
// because of the flag. Nothing faults or traps: the kernel returns and the context stays usable.
#include <cstdint>

#include "mxattn_internal.h"
#include "sm100_ptx.cuh"

namespace mxattn {
namespace {

__global__ void __launch_bounds__(64) wait_timeout_selftest_kernel(unsigned int* status, unsigned int* seen) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);   // phase 0 needs one arrival that never comes
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* flag = &abort_flag;
  if (threadIdx.x < 32) {
    const bool ok = mbar_wait(&bar, 0, flag, status, kStatusSelfTest | 1);
    if (threadIdx.x == 0 && !ok) atomicOr(seen, 1u);
  } else {
    // starts 200 ms after warp 0, so warp 0's bound runs out first and this warp must leave
    // through the abort flag (its own bound would only end 200 ms later)
    const uint64_t t0 = global_timer_ns();
    while (global_timer_ns() - t0 < 200ull * 1000ull * 1000ull) __nanosleep(1000);
    const bool ok = mbar_wait(&bar, 0, flag, status, kStatusSelfTest | 2);
    if (threadIdx.x == 32 && !ok) atomicOr(seen, 2u);
  }
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(unsigned int* status, unsigned int* seen, cudaStream_t stream) {
  wait_timeout_selftest_kernel<<<1, 64, 0, stream>>>(status, seen);
  return cudaGetLastError();
}

}  // namespace mxattn
