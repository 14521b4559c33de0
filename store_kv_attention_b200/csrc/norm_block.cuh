// Per-iteration safety check of one lane by one thread block.
// [Novel Contributions, "Novel: Per-Iteration Safety Check";
//  Architecture-Exclusive Features, "Per-iteration safety check"]
//
// The sum of squares of the lane's fp32 residual row is accumulated in FP64 (each square
// is exact in FP64) and reduced in a fixed order (per-thread strided sums, a butterfly in
// each warp, then the warps in index order), so the result does not depend on scheduling.
// The abort decision is the FP64 comparison n2 > threshold^2; the flag is sticky and the
// first aborting iteration is kept.
#pragma once

#include "tl_internal.cuh"

namespace tl {

template <int kThreadsPerBlock>
__device__ __forceinline__ void norm_check_lane(const float* __restrict__ residual, int b, int d, float threshold,
                                                int iter, uint8_t* flags, int32_t* first, float* norms) {
  static_assert(kThreadsPerBlock % 32 == 0 && kThreadsPerBlock <= 1024, "whole warps");
  __shared__ double warp_sum[kThreadsPerBlock / 32];
  const float* r = residual + (size_t)b * d;
  double acc = 0.0;
  if ((d & 3) == 0 && ((uintptr_t)r & 15) == 0) {
    const float4* r4 = reinterpret_cast<const float4*>(r);
    for (int i = threadIdx.x; i < d / 4; i += kThreadsPerBlock) {
      const float4 v = r4[i];
      acc += (double)v.x * v.x + (double)v.y * v.y + (double)v.z * v.z + (double)v.w * v.w;
    }
  } else {
    for (int i = threadIdx.x; i < d; i += kThreadsPerBlock) acc += (double)r[i] * r[i];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) warp_sum[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double n2 = 0.0;
    for (int w = 0; w < kThreadsPerBlock / 32; ++w) n2 += warp_sum[w];
    const double thr = (double)threshold;
    if (n2 > thr * thr) {
      if (flags[b] == 0) first[b] = iter;
      flags[b] = 1;
    }
    if (norms) norms[b] = (float)sqrt(n2);
  }
}

}  // namespace tl
