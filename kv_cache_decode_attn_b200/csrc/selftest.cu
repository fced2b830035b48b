// Self-test of the library's failure detection: one thread waits, through the
// same bounded wait every warp-specialised kernel here uses, on an mbarrier that
// nothing arrives at.  The wait must give up after its limit and the kernel
// records ATTN_DEV_TIMEOUT in the status word, as a kernel whose wait ran out
// does; the context stays usable.  No trap, no fault, no unbounded loop.
#include "internal.h"
#include "ptx.cuh"

namespace kvattn {
namespace {

__global__ void wait_timeout_kernel(unsigned* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    if (!mbar_wait(&bar, 0)) atomicOr(status, DEV_TIMEOUT);   // phase 0 never completes
  }
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(unsigned* status, cudaStream_t stream) {
  wait_timeout_kernel<<<1, 32, 0, stream>>>(status);
  return cudaGetLastError();
}

}  // namespace kvattn
