// Self-test of the bounded-wait machinery every tensor-core kernel relies
// on: one CTA waits on an mbarrier that nothing will ever arrive on. The
// wait must give up after its cycle budget, record kStTimeout in the device
// status word and return, leaving the context usable.
#include "tc_ptx.cuh"

namespace moba {
namespace {

__global__ void wait_selftest_kernel(int* status, int* done) {
  __shared__ uint64_t bar;
  __shared__ int abort;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);  // one arrival expected; none is made
    abort = 0;
    tc::mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = tc::mbar_wait(&bar, 0, &abort, status);
    *done = ok ? 1 : 2;
  }
}

}  // namespace

cudaError_t launch_wait_selftest(int* status, int* done, cudaStream_t st) {
  wait_selftest_kernel<<<1, 32, 0, st>>>(status, done);
  return cudaGetLastError();
}

}  // namespace moba
