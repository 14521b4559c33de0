/*
 * tl_delta.h -- iteration-axis delta cache of h: layout, writer and decode.
 *
 * [Architecture-Exclusive Features, "Iteration-axis delta-KV"; Measured benchmarks,
 *  "iteration-axis delta-KV: full forward-path PPL A/B"]
 * Along the loop iterations a token's hidden state h contracts, so the cache keeps, per
 * token, one fp16 anchor (the state of loop iteration 0) and, for every later iteration i,
 * an INT8 delta with one fp16 scale per head.  The state of iteration i is rebuilt as
 *     h^i = anchor + sum_{j=1..i} scale_j[head] * code_j        (FP32 prefix sum)
 * This header covers the cache layout, the writer, and a decode over the cache: the new
 * token's state is written, then the store-h decode runs with the FP32 prefix sum as its
 * dequantisation stage, inside the kernel that attends the rows (tl_delta_attn_decode).
 *
 * Conventions are those of tl_storeh.h: caller-owned device memory, asynchronous on a
 * stream, host-side validation before any launch (a non-TL_OK return enqueues nothing,
 * except TL_ERR_CUDA for a failed launch), programmatic dependent launch with stream order
 * preserved, tl_last_error_message() for details.
 */
#ifndef TL_DELTA_H_
#define TL_DELTA_H_

#include "tl_storeh.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Shape of one delta cache (one loop block).  d_model = n_heads * head_dim, head_dim in
 * {64, 128}, d_model a multiple of 256 and at most 2048; L_max loop iterations; max_ctx
 * positions per lane. */
typedef struct {
  int32_t d_model, n_heads, head_dim;
  int32_t L_max;
  int32_t max_lanes;
  int32_t max_ctx;
} tl_delta_desc;

/* Device buffers, caller-allocated, each 256-byte aligned:
 *   anchor [max_lanes][max_ctx][d_model]          fp16  (state of iteration 0)
 *   deltas [L_max-1][max_lanes][max_ctx][d_model]  int8  (iteration i >= 1 at index i-1)
 *   scales [L_max-1][max_lanes][max_ctx][n_heads]  fp16  (one per head, same indexing)
 * deltas and scales may be NULL when L_max == 1. */
typedef struct {
  void* anchor;
  void* deltas;
  void* scales;
} tl_delta_cache;

/* Sizes in bytes of the three buffers for `desc`.
 * Errors: TL_ERR_INVALID_ARG (NULL pointer, non-positive size), TL_ERR_SHAPE
 * (d_model != n_heads * head_dim), TL_ERR_UNSUPPORTED (head_dim or d_model outside the
 * supported set). */
TL_API tl_status tl_delta_cache_bytes(const tl_delta_desc* desc, size_t* anchor_bytes, size_t* delta_bytes,
                                      size_t* scale_bytes);

/* Writes the states of loop iteration `iter` of n_rows positions per lane.
 *   h_rows    device fp16 [n_lanes][n_rows][d_model], 16-byte aligned: h^iter of each row
 *   start_pos device int32 [n_lanes]: row r of lane b goes to position start_pos[b] + r
 *   loops     device int32 [n_lanes] or NULL: lane b is skipped when iter >= loops[b]
 * iter == 0 stores the rows as the anchor.  iter >= 1 first rebuilds h^(iter-1) of each
 * position from the cache in FP32 (anchor, then iterations 1..iter-1 added in order, each
 * addition rounded to fp32) and stores dh = h^iter - that rebuild, per head:
 *   scale = fp16_rne(amax / 127.0f)  (fp32 IEEE division, amax = max |dh| over the head)
 *   code  = clamp(rne(dh / float(scale)), -127, 127)  (fp32 IEEE division; zero scale ->
 *           zero codes)
 * so the rebuild error of iteration i is that of its own delta only.  Iterations of a
 * position must therefore be written in order.  Rows whose position lies outside
 * [0, max_ctx) are skipped on the device.
 * Errors: TL_ERR_INVALID_ARG (NULL or misaligned pointer, bad count), TL_ERR_CAPACITY
 * (n_lanes > max_lanes, iter outside [0, L_max)), the desc errors above, TL_ERR_CUDA. */
TL_API tl_status tl_delta_append(const tl_delta_desc* desc, tl_delta_cache cache, int32_t iter, const void* h_rows,
                                 int32_t n_lanes, int32_t n_rows, const int32_t* start_pos, const int32_t* loops,
                                 tl_stream_t stream);

/* Workspace bytes of tl_delta_attn_decode for n_lanes lanes: the store-h decode workspace
 * (status word first) in the layout of 256-row splits with hi and lo absorbed-query images,
 * plus two int32 [n_lanes] arrays of per-lane loop flags.  The rebuilt states are never
 * stored.
 * Errors: the desc errors, TL_ERR_INVALID_ARG (n_lanes <= 0, NULL), TL_ERR_CAPACITY
 * (n_lanes > max_lanes), TL_ERR_UNSUPPORTED (n_lanes > 64, n_heads > 16, max_ctx > 65536). */
TL_API tl_status tl_delta_workspace_bytes(const tl_delta_desc* desc, int32_t n_lanes, size_t* bytes);

/* Decode attention of loop iteration `iter` over the delta cache, one new token per lane.
 * Arguments as for tl_storeh_append_attn_decode (tl_storeh.h): loops / ctx_len device int32
 * [n_lanes]; h_new fp16 [n_lanes][d] = the new token's state of iteration iter; W_q, W_k, W_v
 * fp16 [d][d]; out fp32 [n_lanes][d]; the optional safety check (residual fp32 [n_lanes][d],
 * threshold, abort_flags, first_abort_iter, norms_out); workspace of
 * tl_delta_workspace_bytes bytes, 256-byte aligned, its first 256 bytes zeroed once.
 * For every lane with iter < loops[b] (a lane whose loops / ctx_len are out of range is
 * skipped and recorded; tl_storeh_poll_status on this workspace reports it):
 *   1. h_new is written as the state of iteration iter at position ctx_len[b], exactly as
 *      tl_delta_append does;
 *   2. q = W_q h_new attends positions 0..ctx_len[b] with K = W_k h, V = W_v h (the
 *      store-h decode), where each attended row h^iter is rebuilt inside the streaming
 *      kernel by the FP32 prefix sum above and enters the tensor cores as an fp16 hi + lo
 *      pair per value (about 22 significant bits), the absorbed query and the softmax
 *      weights likewise;
 *   3. with a residual, the safety check of iteration iter runs as in tl_residual_norm_check.
 * Other lanes' out rows are left unwritten.  Errors: as tl_storeh_attn_decode, plus the
 * desc errors above, and TL_ERR_UNSUPPORTED for n_heads > 16.
 * Accuracy: against the FP64 rebuild and attention, outputs meet the store-h bar (max-abs
 * 2e-3, relative L2 1e-3) in the seeded GPU tests at d_model 256, 768, 1024 (3 and 8 loop
 * iterations), 1280 and 2048. */
TL_API tl_status tl_delta_attn_decode(const tl_delta_desc* desc, tl_delta_cache cache, int32_t iter,
                                      const int32_t* loops, const int32_t* ctx_len, const void* h_new,
                                      const void* W_q, const void* W_k, const void* W_v, float* out,
                                      const float* residual, float threshold, uint8_t* abort_flags,
                                      int32_t* first_abort_iter, float* norms_out, void* workspace,
                                      size_t workspace_bytes, int32_t n_lanes, tl_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* TL_DELTA_H_ */
