// Quantisation of one fp16 h row into the store-h cache, by every thread of a block.
// [Architecture-Exclusive Features, "Store-h KV cache" (FP16-h / INT8-h / INT4-h modes)]
//
// Codes are bit-exact with the format definitions in tl_storeh.h: the scale is an IEEE fp32
// division of the absolute maximum, every code an IEEE fp32 division rounded half to even, then
// clamped.  Used by the append kernel and by the fused append of the decode's q projection.
#pragma once

#include <cuda_fp16.h>

#include "tl_internal.cuh"

namespace tl {

__device__ __forceinline__ float row_warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ int quant_code(float x, float div, int qmax) {
  if (div == 0.0f) return 0;
  int c = __float2int_rn(__fdiv_rn(x, div));  // IEEE division, round half to even
  return max(-qmax, min(qmax, c));
}

// Writes row `row` (index into the cache's rows) from `src` (d fp16 values).  Every thread of
// the block calls it (INT8 takes a block-wide maximum).
template <int kThreads>
__device__ void append_row_block(const Shape& s, uint8_t* codes, uint8_t* scales, size_t row, const __half* src) {
  const int d = s.d;
  if (s.fmt == TL_H_FP16) {
    const uint4* in = reinterpret_cast<const uint4*>(src);
    uint4* out = reinterpret_cast<uint4*>(codes + row * (size_t)(2 * d));
    for (int i = threadIdx.x; i < d / 8; i += kThreads) out[i] = in[i];
    return;
  }

  if (s.fmt == TL_H_INT8_TOKEN) {
    __shared__ float red[kThreads / 32];
    float amax = 0.0f;
    for (int i = threadIdx.x; i < d; i += kThreads) amax = fmaxf(amax, fabsf(__half2float(src[i])));
    amax = row_warp_max(amax);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int w = 1; w < kThreads / 32; ++w) amax = fmaxf(amax, red[w]);
    __syncthreads();  // red is free again once every thread has read it
    const float scale = __fdiv_rn(amax, 127.0f);
    int8_t* out = reinterpret_cast<int8_t*>(codes + row * (size_t)d);
    for (int i = threadIdx.x; i < d; i += kThreads) out[i] = (int8_t)quant_code(__half2float(src[i]), scale, 127);
    if (threadIdx.x == 0) reinterpret_cast<float*>(scales)[row] = scale;
    return;
  }

  // INT4, groups of 64: one warp per group, two elements per lane -> one byte per lane.
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  uint8_t* out = codes + row * (size_t)(d / 2);
  __half* sc = reinterpret_cast<__half*>(scales) + row * (size_t)(d / kInt4Group);
  for (int g = warp; g < d / kInt4Group; g += kThreads / 32) {
    const __half2 v = reinterpret_cast<const __half2*>(src + g * kInt4Group)[lane];
    const float x0 = __low2float(v), x1 = __high2float(v);
    const float amax = row_warp_max(fmaxf(fabsf(x0), fabsf(x1)));
    const __half s16 = __float2half_rn(__fdiv_rn(amax, 7.0f));
    const float div = __half2float(s16);
    const int c0 = quant_code(x0, div, 7), c1 = quant_code(x1, div, 7);
    out[g * (kInt4Group / 2) + lane] = (uint8_t)((c0 & 0xF) | ((c1 & 0xF) << 4));
    if (lane == 0) sc[g] = s16;
  }
}

}  // namespace tl
