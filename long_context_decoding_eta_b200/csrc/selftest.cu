// Diagnostics.  The wait test proves on the device that a pipeline wait that never
// completes ends by itself with a status the host can read, leaving the context
// usable; the bounds test runs the checked build's range check on a given index
// (no memory access), so that its reporting path can be exercised.
// The kernel waits, with the same bounded wait the decode kernels use, on an
// mbarrier that nothing ever arrives on, and on a global flag that nothing sets.
#include "eta_common.cuh"
#include "eta_host.h"

namespace eta {

__global__ void selftest_wait_kernel(uint32_t limit, const volatile int32_t* never_set,
                                     int32_t* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  if (!mbar_wait_n(&bar, 0, nullptr, limit)) set_status(status, ETA_DEVSTAT_TIMEOUT);
  if (never_set) {
    uint32_t i = 0;
    while (i < limit && *never_set == 0) ++i;
    if (i == limit) set_status(status, ETA_DEVSTAT_TIMEOUT);
  }
}

__global__ void selftest_bounds_kernel(long long index, long long extent, int32_t* status) {
  (void)ETA_IN_BOUNDS(index, extent, status);
  (void)status;
}

}  // namespace eta

extern "C" int32_t eta_build_checked(void) { return eta::kChecked ? 1 : 0; }

extern "C" eta_status_t eta_selftest_bounds(int64_t index, int64_t extent, int32_t* dev_status,
                                            void* stream) {
  if (!dev_status || extent < 0) return ETA_ERR_INVALID_ARG;
  eta::selftest_bounds_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(
      (long long)index, (long long)extent, dev_status);
  return eta::launch_status();
}

extern "C" eta_status_t eta_selftest_wait_timeout(uint32_t wait_limit, const int32_t* never_set,
                                                  int32_t* dev_status, void* stream) {
  if (!dev_status || wait_limit == 0 || wait_limit > (1u << 24)) return ETA_ERR_INVALID_ARG;
  eta::selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      wait_limit, never_set, dev_status);
  return eta::launch_status();
}
