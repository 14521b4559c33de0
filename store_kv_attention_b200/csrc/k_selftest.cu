// Self-test of the failure-detection path: a kernel whose only wait can never complete (an
// mbarrier nothing arrives at), bounded by the same helper every kernel of the library uses.
// It gives up after `limit` SM clocks and records kStatusTimeout in the status word, exactly as
// a kernel that timed out in earnest does; tl_storeh_poll_status then reports it.
#include "tc_ptx.cuh"
#include "tl_internal.cuh"

namespace tl {
namespace {

__global__ void wait_selftest_kernel(uint32_t* status, long long limit) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  ptx::mbar_init(&bar, 1);
  ptx::mbar_fence_init();
  abort_flag = 0;
  if (!ptx::mbar_wait(&bar, 0, (volatile int*)&abort_flag, limit)) atomicOr(status, kStatusTimeout);
}

}  // namespace

cudaError_t launch_wait_selftest(uint32_t* status, long long limit_cycles, cudaStream_t st) {
  wait_selftest_kernel<<<1, 32, 0, st>>>(status, limit_cycles);
  count_launch();
  return cudaGetLastError();
}

}  // namespace tl
