// Per-iteration safety check on the residual L2 norm (standalone entry point).
// [Novel Contributions, "Novel: Per-Iteration Safety Check";
//  Architecture-Exclusive Features, "Per-iteration safety check"]
//
// One thread block per lane (norm_block.cuh); the decode call runs the same routine
// inside its merge kernel.
#include "norm_block.cuh"
#include "tc_ptx.cuh"

namespace tl {
namespace {

constexpr int kNormThreads = 256;

__global__ void __launch_bounds__(kNormThreads) norm_kernel(const float* __restrict__ residual, int d, float threshold,
                                                            int iter, const int32_t* __restrict__ loops,
                                                            uint8_t* flags, int32_t* first, float* norms) {
  ptx::pdl_wait();  // the residual may come from the previous kernel in the stream
  ptx::pdl_trigger();
  const int b = blockIdx.x;
  if (loops && iter >= loops[b]) return;
  norm_check_lane<kNormThreads>(residual, b, d, threshold, iter, flags, first, norms);
}

}  // namespace

cudaError_t launch_norm_check(const float* residual, int n_lanes, int d, float threshold, int iter,
                              const int32_t* loops, uint8_t* flags, int32_t* first, float* norms, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_lanes, 1, 1);
  cfg.blockDim = dim3(kNormThreads, 1, 1);
  cfg.stream = st;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, norm_kernel, residual, d, threshold, iter, loops, flags, first, norms);
  count_launch();
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace tl
