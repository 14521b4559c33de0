// Append: quantise fp16 h rows into the store-h cache.
// [Architecture-Exclusive Features, "Store-h KV cache" (FP16-h / INT8-h / INT4-h
//  modes); "Variable-L KV cache" (layer n_pre+i is written by loop iteration i)]
//
// One CTA of 128 threads per (row, lane); the row itself is quantised by append_row_block
// (append_row.cuh).
#include "append_row.cuh"
#include "tc_ptx.cuh"
#include "tl_internal.cuh"

namespace tl {
namespace {

constexpr int kThreads = 128;

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
  append_row_block<kThreads>(s, codes, scales, row, h_rows + ((size_t)b * n_rows + r) * s.d);
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
