// Diagnostic: exercise the bounded device-side wait on a barrier that nothing
// ever completes.  The waiting thread must give up after the limit, raise
// LRMOE_ST_TIMEOUT in the status word and return, leaving the context usable.
#include "common.cuh"
#include "launch.h"

namespace lrmoe {
namespace {

__global__ void bounded_wait_kernel(uint64_t limit_ns, uint32_t* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // one arrival would complete phase 0; none ever comes
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = mbar_wait_bounded(&bar, 0, &abort_flag, status, limit_ns);
    if (ok) raise_status(status, LRMOE_ST_BAD_INDEX);  // cannot happen: nobody arrived
  }
}

}  // namespace

cudaError_t launch_selftest_wait(uint32_t limit_us, uint32_t* status, cudaStream_t s) {
  bounded_wait_kernel<<<1, 32, 0, s>>>((uint64_t)limit_us * 1000ull, status);
  return cudaGetLastError();
}

}  // namespace lrmoe
