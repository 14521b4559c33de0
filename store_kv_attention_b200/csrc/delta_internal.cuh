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

// One delta decode call (tl_delta_attn_decode): per-lane effective loop counts for the writer
// and the decode, range violations recorded in *status.
cudaError_t launch_delta_prep(int iter, int L_max, int max_ctx, int n_lanes, const int32_t* loops,
                              const int32_t* ctx_len, int32_t* wloops, int32_t* dloops, uint32_t* status,
                              cudaStream_t st);
struct Workspace;
// The decode's streaming stage over the delta cache (k_delta_stream.cu): rows 0..ctx_len[b] of
// every lane with dloops[b] = 1 rebuilt by the FP32 prefix sum of levels 1..iter, attended with
// the absorbed-query images of the decode workspace `ws` (layout wl), split partials into ws.
cudaError_t launch_delta_stream(const DeltaShape& s, const void* anchor, const void* deltas, const void* scales,
                                int iter, int n_lanes, const int32_t* dloops, const int32_t* ctx_len, uint8_t* ws,
                                const Workspace& wl, cudaStream_t st);

}  // namespace tl
