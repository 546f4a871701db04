// Failure-detection self-test kernel (declared in selftest.cuh).
#include "kernels.cuh"
#include "ptx.cuh"
#include "selftest.cuh"

namespace i8mm {
namespace {

__global__ void wait_selftest_kernel(const uint32_t* flag, int* status, unsigned long long timeout_ns) {
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1; ld_acquire_gpu_u32(flag) == 0u; ++it) {
    if ((it & 15u) == 0 && global_timer_ns() - t0 > timeout_ns) {
      atomicOr(status, kStatusTimeout);
      return;
    }
  }
}

}  // namespace

cudaError_t launch_wait_selftest(const uint32_t* flag, int* status, unsigned long long timeout_ns,
                                 cudaStream_t stream) {
  wait_selftest_kernel<<<1, 1, 0, stream>>>(flag, status, timeout_ns);
  return cudaGetLastError();
}

}  // namespace i8mm
