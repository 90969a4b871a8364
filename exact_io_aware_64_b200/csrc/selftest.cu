// selftest.cu -- a deliberately unsatisfied, bounded wait, to check the failure path.
//
// Every pipeline wait in the attention kernels spins on an mbarrier with a time limit;
// when the limit runs out the kernel sets kErrWaitTimeout in the library's error word,
// raises its CTA's abort flag and returns, and fa_check_device_error reports
// FA_ERR_TIMEOUT.  This probe waits on a barrier that nothing ever arrives on, with the
// same loop form and a caller-chosen limit, so that path can be exercised on purpose:
// the kernel ends by itself after about `limit` cycles and the context stays usable.
#include <cstdint>

#include "internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

using namespace sm100;

__global__ void __launch_bounds__(32) timeout_probe_kernel(unsigned int* err, long long limit) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // phase 0 of a fresh barrier with one expected arrival completes only when something
  // arrives: nothing does
  const long long t0 = clock64();
  uint32_t spins = 0;
  while (!mbar_try_wait(b, 0)) {
    if (++spins % kSpinCheck == 0) {
      if (*static_cast<volatile int*>(&abort_flag)) break;
      if (clock64() - t0 > limit) {
        atomicOr(err, kErrWaitTimeout);
        abort_flag = 1;
        break;
      }
    }
  }
  __syncthreads();
}

}  // namespace

cudaError_t launch_timeout_probe(long long limit_cycles, const Problem& p,
                                 cudaStream_t stream) {
  timeout_probe_kernel<<<1, 32, 0, stream>>>(p.err, limit_cycles);
  return cudaGetLastError();
}

}  // namespace fa
