// Append: quantise fp16 h rows into the store-h cache.
// [Architecture-Exclusive Features, "Store-h KV cache" (FP16-h / INT8-h / INT4-h
//  modes); "Variable-L KV cache" (layer n_pre+i is written by loop iteration i)]
//
// One CTA of 128 threads per (row, lane).  Codes are bit-exact with the format
// definitions in tl_storeh.h: the scale is an IEEE fp32 division of the absolute
// maximum, every code an IEEE fp32 division rounded half to even, then clamped.
#include "tc_ptx.cuh"
#include "tl_internal.cuh"

namespace tl {
namespace {

constexpr int kThreads = 128;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ int quant_code(float x, float div, int qmax) {
  if (div == 0.0f) return 0;
  int c = __float2int_rn(__fdiv_rn(x, div));  // IEEE division, round half to even
  return max(-qmax, min(qmax, c));
}

__global__ void __launch_bounds__(kThreads) append_kernel(Shape s, uint8_t* codes, uint8_t* scales, int layer,
                                                          const __half* __restrict__ h_rows, int n_rows,
                                                          const int32_t* __restrict__ start_pos,
                                                          const int32_t* __restrict__ row_count,
                                                          const int32_t* __restrict__ loops) {
  ptx::pdl_wait();  // the rows may come from the previous kernel in the stream
  ptx::pdl_trigger();
  const int r = blockIdx.x;
  const int b = blockIdx.y;
  if (loops && layer >= s.n_pre + loops[b]) return;
  if (row_count && r >= row_count[b]) return;
  const long long pos = (long long)start_pos[b] + r;
  if (pos < 0 || pos >= s.max_ctx) return;
  const size_t row = ((size_t)layer * s.max_lanes + b) * s.max_ctx + (size_t)pos;
  const __half* src = h_rows + ((size_t)b * n_rows + r) * s.d;
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
    amax = warp_max(amax);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int w = 1; w < kThreads / 32; ++w) amax = fmaxf(amax, red[w]);
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
    const float amax = warp_max(fmaxf(fabsf(x0), fabsf(x1)));
    const __half s16 = __float2half_rn(__fdiv_rn(amax, 7.0f));
    const float div = __half2float(s16);
    const int c0 = quant_code(x0, div, 7), c1 = quant_code(x1, div, 7);
    out[g * (kInt4Group / 2) + lane] = (uint8_t)((c0 & 0xF) | ((c1 & 0xF) << 4));
    if (lane == 0) sc[g] = s16;
  }
}

}  // namespace

cudaError_t launch_append(const Shape& s, void* codes, void* scales, int layer, const __half* h_rows, int n_lanes,
                          int n_rows, const int32_t* start_pos, const int32_t* row_count, const int32_t* loops,
                          cudaStream_t st) {
  if (n_lanes > 65535) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_rows, n_lanes, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.stream = st;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, append_kernel, s, (uint8_t*)codes, (uint8_t*)scales, layer, h_rows, n_rows,
                                     start_pos, row_count, loops);
  count_launch();
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace tl
