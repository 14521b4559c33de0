// Internal declarations shared by the host API and the kernels of libtlstoreh.so.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "tl_storeh.h"

namespace tl {

// ---------------------------------------------------------------- status word bits
// The first 256 bytes of the decode workspace hold the device status word.
enum : uint32_t {
  kStatusRange = 1u << 0,    // a lane's loops / ctx_len was out of range; the lane was skipped
  kStatusTimeout = 1u << 1,  // a bounded wait gave up
};

constexpr int kInt4Group = 64;
constexpr int kMaxHeads = 16;        // heads are padded to 16 in the kernels
constexpr int kSplitRows = 1024;     // default context rows per split (a call may choose 128, 256, 512 or 1024)
constexpr int kMaxCtx = 65536;       // positions per (layer, lane) the kernels support
constexpr int kDeltaSplitRows = 256;  // context rows per split of the delta-cache decode
constexpr int kMaxSplits = kMaxCtx / kSplitRows;

// ---------------------------------------------------------------- shapes
struct Shape {
  int d, H, hd, n_pre, L_max, max_lanes, max_ctx, fmt;
  __host__ __device__ int layers() const { return n_pre + L_max; }
  __host__ __device__ size_t row_code_bytes() const {
    return fmt == TL_H_FP16 ? 2 * (size_t)d : fmt == TL_H_INT8_TOKEN ? (size_t)d : (size_t)d / 2;
  }
  __host__ __device__ int row_scales() const { return fmt == TL_H_FP16 ? 0 : fmt == TL_H_INT8_TOKEN ? 1 : d / kInt4Group; }
  __host__ __device__ size_t scale_bytes() const { return fmt == TL_H_INT8_TOKEN ? 4 : 2; }
  __host__ __device__ size_t rows_total() const { return (size_t)layers() * max_lanes * max_ctx; }
};

// Operand precision of the tensor-core path: when d <= 1024 the absorbed query and
// P are split into fp16 hi + lo parts (32 MMA columns instead of 16).
__host__ __device__ inline bool split_operands(int d) { return d <= 1024; }
__host__ __device__ inline int qimg_rows(int d) { return split_operands(d) ? 32 : 16; }
__host__ __device__ inline size_t qimg_bytes(int d) { return (size_t)qimg_rows(d) * d * 2; }

// Physical K position of logical d-index c in the dequantised operand order.
// INT4 words are unpacked as pairs (e0,e4),(e1,e5),(e2,e6),(e3,e7): position p of a
// group of 8 holds element (p >> 1) + 4 * (p & 1), so element e sits at 2 * (e & 3) + (e >> 2).
__host__ __device__ inline int phys_pos(int fmt, int c) {
  if (fmt != TL_H_INT4_G64) return c;
  const int e = c & 7;
  return (c & ~7) + 2 * (e & 3) + (e >> 2);
}
__host__ __device__ inline int logical_of_pos(int fmt, int pos) {
  if (fmt != TL_H_INT4_G64) return pos;
  const int p = pos & 7;
  return (pos & ~7) + (p >> 1) + 4 * (p & 1);
}

// Byte offset of K-position `pos` of row `row` in a K-major, 128-byte-swizzled fp16
// operand made of atom-columns of 64 values, each atom-column `rows` high
// (the canonical layout of a UMMA operand with SWIZZLE_128B).
__host__ __device__ inline uint32_t kmajor_offset(int row, int pos, int rows) {
  const int a = pos >> 6, c = pos & 63;
  return (uint32_t)(a * rows * 128 + row * 128 + ((((c >> 3) ^ (row & 7)) << 4) | ((c & 7) << 1)));
}

__host__ __device__ inline int splits_for_rows(int n_rows, int split = kSplitRows) { return (n_rows + split - 1) / split; }
__host__ __device__ inline bool valid_split_rows(int split) {
  return split == 128 || split == 256 || split == 512 || split == 1024;
}

// Rows a (virtual) lane attends, for multi-query calls (tree verification, chunked prefill):
// rows [0, n0) and [start1, start1 + n1) of physical lane `phys` in the iteration's layer.
// Each segment is cut into splits of kSplitRows rows of its own, segment 0's first, so a split
// is one contiguous run of rows.  A decode lane b is {b, ctx_len[b] + 1, 0, 0}.
struct LaneSeg {
  int32_t phys, n0, start1, n1;
};
__host__ __device__ inline int seg_splits(const LaneSeg& g, int split) {
  return splits_for_rows(g.n0, split) + splits_for_rows(g.n1, split);
}
// Split `split_idx` of a lane (splits of `split` rows): first row (in the physical lane's row
// space) and row count; false when the lane has fewer splits.
__host__ __device__ inline bool seg_split_rows(const LaneSeg& g, int split_idx, int split, int* r_begin, int* n_rows) {
  const int s0 = splits_for_rows(g.n0, split);
  if (split_idx < s0) {
    *r_begin = split_idx * split;
    *n_rows = g.n0 - *r_begin < split ? g.n0 - *r_begin : split;
    return true;
  }
  const int s1 = split_idx - s0;
  if (s1 * split >= g.n1) return false;
  *r_begin = g.start1 + s1 * split;
  *n_rows = g.n1 - s1 * split < split ? g.n1 - s1 * split : split;
  return true;
}

// ---------------------------------------------------------------- decode-step geometry
constexpr int kMaxGemmLanes = 64;  // lanes per decode call (projection MMAs with N <= 256, 64-bit lane masks)

__host__ __device__ inline int lanes_padded(int n_lanes) { return (n_lanes + 15) & ~15; }

// Whether lane b takes part in iteration `iter` (loops / ctx_len in range and iter < loops[b]);
// n_rows = the lane's cached positions plus the new one.
__device__ __forceinline__ bool lane_active(const Shape& s, int iter, const int32_t* loops, const int32_t* ctx_len,
                                            int b, int* n_rows) {
  const int L = loops[b];
  const int c = ctx_len[b];
  if (L < 0 || L > s.L_max || c < 0 || c >= s.max_ctx) return false;
  if (iter >= L) return false;
  *n_rows = c + 1;
  return true;
}

// ---------------------------------------------------------------- workspace layout
// All offsets are 256-byte aligned.
struct Workspace {
  size_t status_off;   // uint32 status word (+ padding to 256 bytes)
  size_t qt_off;       // fp16 [n_lanes][qrows x d] absorbed query operand images (stream kernel)
  size_t ml_off;       // fp32 [n_lanes][S_max][16][2]   per-split running max and sum
  size_t u_off;        // fp32 [n_lanes][S_max][16][d]   per-split unnormalised sum_c p_c h_c
  size_t total;
  int s_max, nb;
  int split;           // context rows per split
  int qrows;           // rows of a query image: 16 (fp16) or 32 (fp16 hi + lo)
};

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// extra_splits: splits a lane may have beyond those of max_ctx rows in one run (multi-query
// calls, whose second row segment starts a split of its own).
// qt_split: hi / lo query images at every d (otherwise only where split_operands(d)).
inline Workspace workspace_layout(const Shape& s, int n_lanes, int extra_splits = 0, int split = kSplitRows,
                                  bool qt_split = false) {
  Workspace w;
  w.split = split;
  w.qrows = (qt_split || split_operands(s.d)) ? 32 : 16;
  w.s_max = splits_for_rows(s.max_ctx, split) + extra_splits;
  w.nb = lanes_padded(n_lanes);
  size_t off = 0;
  w.status_off = off;
  off += 256;
  w.qt_off = off;
  off = align256(off + (size_t)n_lanes * w.qrows * (size_t)s.d * 2);
  w.ml_off = off;
  off = align256(off + (size_t)n_lanes * w.s_max * kMaxHeads * 2 * 4);
  w.u_off = off;
  off = align256(off + (size_t)n_lanes * w.s_max * kMaxHeads * (size_t)s.d * 4);
  w.total = off;
  return w;
}

// Launch attribute for programmatic dependent launch: the kernel may be scheduled while the previous
// kernel in the stream drains, and waits for it (griddepcontrol.wait) before touching global memory.
inline cudaLaunchAttribute pdl_attribute() {
  cudaLaunchAttribute a;
  a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a.val.programmaticStreamSerializationAllowed = 1;
  return a;
}

// Records a message for tl_last_error_message() and returns `st`.
tl_status set_error(tl_status st, const char* fmt, ...);

// ---------------------------------------------------------------- measurement hook
tl_profile*& current_profile();                  // thread-local; NULL when not installed
inline void count_launch(int n = 1) {
  if (tl_profile* p = current_profile()) p->launches += n;
}
void profile_stream_begin(cudaStream_t st);      // records begin_events[recorded] if installed
void profile_stream_end(cudaStream_t st);        // records end_events[recorded++] if installed

// ---------------------------------------------------------------- kernel launch limits
// The largest dynamic shared memory a launch of `func` may request on the current device.  The
// kernel is opted into it (cudaFuncAttributeMaxDynamicSharedMemorySize = the device's per-block
// opt-in limit minus the kernel's static shared memory) the first time, and the limit is cached
// per (kernel, device), so a decode call costs no attribute queries after the first (tl_api.cu).
cudaError_t dyn_smem_limit(const void* func, int* limit);

// ---------------------------------------------------------------- launchers (return cudaError_t)
cudaError_t launch_append(const Shape& s, void* codes, void* scales, int layer, const __half* h_rows,
                          int n_lanes, int n_rows, const int32_t* start_pos, const int32_t* row_count,
                          const int32_t* loops, cudaStream_t st);

// Standalone safety check of tl_residual_norm_check (lanes with iter >= loops[b] skipped when loops is given).
cudaError_t launch_norm_check(const float* residual, int n_lanes, int d, float threshold, int iter,
                              const int32_t* loops, uint8_t* flags, int32_t* first, float* norms, cudaStream_t st);

struct DecodeArgs {
  Shape s;
  const void* codes;
  const void* scales;
  int iter;
  const int32_t* loops;
  const int32_t* ctx_len;
  const __half* h_new;
  const __half* Wq;
  const __half* Wk;
  const __half* Wv;
  float* out;
  int n_lanes;
  uint8_t* ws;
  Workspace wl;
  // per-iteration safety check fused into the decode (residual == NULL: none)
  const float* residual;
  float threshold;
  uint8_t* abort_flags;
  int32_t* first_abort_iter;
  float* norms;
  // append h_new as the new token's row of every active lane first (fused into qproj_kernel)
  bool append = false;
  // multi-query calls: the rows of each (virtual) lane (device [n_lanes]); NULL = decode lanes
  const LaneSeg* seg = nullptr;
  // RoPE variant: scores computed before the streaming kernel (device fp32 [n_lanes][max_ctx][16])
  const float* scores = nullptr;
};

// Fused q and absorbed-query projections, one thread-block cluster per 128 rows of W_q (k_proj_tc.cu).
cudaError_t launch_qproj(const DecodeArgs& a, cudaStream_t st);
// Fused split merge, value projection and safety check on thread-block clusters (k_proj_tc.cu).
cudaError_t launch_oproj(const DecodeArgs& a, cudaStream_t st);
int proj_cluster(int d);
size_t oproj_smem_bytes(const Shape& s, int n_lanes, int s_max);

// fp16 2D tensor map [rows][cols] (row pitch `pitch_elems`), box [box_cols x box_rows], 128-byte swizzle
// (k_proj_tc.cu).
bool make_tmap_f16(void* tmap, const void* base, uint64_t rows, uint64_t cols, uint64_t pitch_elems,
                   uint32_t box_cols, uint32_t box_rows);
cudaError_t launch_stream(const DecodeArgs& a, cudaStream_t st);
// RoPE variant (k_rope.cu): cos / sin table [hd/2][max_ctx] (angle index major), rotated queries [n_lanes][d] and the
// scores [n_lanes][max_ctx][16] the streaming kernel then takes (DecodeArgs::scores).
cudaError_t launch_rope_scores(const DecodeArgs& a, float rope_base, float2* cs, float* qrot, float* scores,
                               cudaStream_t st);
// Self-test of the timeout path: one wait that cannot complete, bounded by limit_cycles (k_selftest.cu).
cudaError_t launch_wait_selftest(uint32_t* status, long long limit_cycles, cudaStream_t st);

}  // namespace tl
