// Failure-detection self-test: one bounded device wait that runs out.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace i8mm {

// Launches one single-thread kernel that polls `flag` (a device word that
// nothing sets; it must be 0) with an acquire load, the way the forward's
// kernels wait on a ticket or a barrier, bounded by %globaltimer after
// `timeout_ns`.  When the wait runs out it sets kStatusTimeout in `status`
// and returns; it issues no asynchronous copies, so giving up is safe.
cudaError_t launch_wait_selftest(const uint32_t* flag, int* status, unsigned long long timeout_ns,
                                 cudaStream_t stream);

}  // namespace i8mm
