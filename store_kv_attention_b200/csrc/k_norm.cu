// Per-iteration safety check on the residual L2 norm.
// [Novel Contributions, "Novel: Per-Iteration Safety Check";
//  Architecture-Exclusive Features, "Per-iteration safety check"]
//
// One warp per lane; the sum of squares is accumulated in FP64 (every term
// exact), so the abort decision is the same FP64 comparison n2 > thr^2 the
// definition states.
#include "tl_internal.cuh"

namespace tl {
namespace {

constexpr int kWarps = 4;

__global__ void __launch_bounds__(kWarps * 32) norm_kernel(const float* __restrict__ residual, int n_lanes, int d,
                                                           float threshold, int iter,
                                                           const int32_t* __restrict__ loops,
                                                           const int32_t* __restrict__ ctx_len, int max_ctx,
                                                           int L_max, uint8_t* flags, int32_t* first, float* norms) {
  const int b = blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (b >= n_lanes) return;
  if (loops && iter >= loops[b]) return;
  if (ctx_len) {  // fused into decode: lanes the decode skipped as out of range are left untouched
    const int L = loops[b], c = ctx_len[b];
    if (L < 0 || L > L_max || c < 0 || c >= max_ctx) return;
  }
  const float* r = residual + (size_t)b * d;
  double acc = 0.0;
  if ((d & 3) == 0 && ((uintptr_t)residual & 15) == 0) {
    const float4* r4 = reinterpret_cast<const float4*>(r);
    for (int i = lane; i < d / 4; i += 32) {
      const float4 v = r4[i];
      acc += (double)v.x * v.x + (double)v.y * v.y + (double)v.z * v.z + (double)v.w * v.w;
    }
  } else {
    for (int i = lane; i < d; i += 32) acc += (double)r[i] * r[i];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) {
    const double thr = (double)threshold;
    if (acc > thr * thr) {
      if (flags[b] == 0) first[b] = iter;
      flags[b] = 1;
    }
    if (norms) norms[b] = (float)sqrt(acc);
  }
}

}  // namespace

cudaError_t launch_norm_check(const float* residual, int n_lanes, int d, float threshold, int iter,
                              const int32_t* loops, const int32_t* ctx_len, int max_ctx, int L_max, uint8_t* flags,
                              int32_t* first, float* norms, cudaStream_t st) {
  const int blocks = (n_lanes + kWarps - 1) / kWarps;
  norm_kernel<<<blocks, kWarps * 32, 0, st>>>(residual, n_lanes, d, threshold, iter, loops, ctx_len, max_ctx, L_max,
                                              flags, first, norms);
  count_launch();
  return cudaGetLastError();
}

}  // namespace tl
