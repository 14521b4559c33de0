// Internal interface of the iteration-axis delta cache writer (k_delta.cu); the C ABI is
// include/tl_delta.h.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace tl {

struct DeltaShape {
  int d, H, hd;
  int L_max, max_lanes, max_ctx;
};

cudaError_t launch_delta_append(const DeltaShape& s, void* anchor, void* deltas, void* scales, int iter,
                                const __half* h_rows, int n_lanes, int n_rows, const int32_t* start_pos,
                                const int32_t* loops, cudaStream_t st);

}  // namespace tl
