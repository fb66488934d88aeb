// qamw_selftest.cu -- a test hook for failure detection (no counterpart in the
// QAM-W page): a kernel that waits on an mbarrier no one arrives on, with the
// bounded wait the TMA decode uses, so tests can check that a wait that runs
// out reports QAMW_STATUS_TIMEOUT through the status word and leaves the
// context usable, without hanging or faulting the GPU.
#include "qamw_device.cuh"
#include "qamw_internal.h"
#include "qamw_mbarrier.cuh"

namespace qamw {
namespace {

__global__ void wait_timeout_kernel(uint32_t tries, int32_t *status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  // phase 0 of `bar` needs one arrival that never comes
  const bool ok = mbar_wait(&bar, 0u, tries);
  const bool all = __all_sync(0xffffffffu, ok);
  if (!all && threadIdx.x == 0) status_or(status, QAMW_STATUS_TIMEOUT);
}

}  // namespace

cudaError_t launch_wait_timeout(uint32_t tries, int32_t *status, cudaStream_t s) {
  wait_timeout_kernel<<<1, 32, 0, s>>>(tries, status);
  return cudaGetLastError();
}

}  // namespace qamw
