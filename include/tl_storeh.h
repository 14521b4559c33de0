/*
 * tl_storeh.h — C ABI of the store-h decode-attention library (libtlstoreh.so).
 *
 * The method (TinyLoop documentation pages):
 *   - Store-h KV cache: the cache keeps the pre-QKV LayerNorm output h of every
 *     (layer, token) instead of K and V; attention rebuilds K = W_k h and
 *     V = W_v h with the loop block's shared weights.
 *     [Novel Contributions, "Novel Mechanism: Store-h KV Cache";
 *      Architecture-Exclusive Features, "Store-h KV cache"]
 *   - Storage modes FP16-h, INT8-h, INT4-h [same section, mode table].
 *   - Variable-L cache of n_pre + L_max layers; loop iteration i uses layer
 *     n_pre + i; a call with loop count L reads only the first n_pre + L layers.
 *     [Architecture-Exclusive Features, "Variable-L KV cache"]
 *   - L-aware batching: every lane of one batch runs its own loop count.
 *     [Architecture-Exclusive Features, "L-aware batching"]
 *   - Per-iteration safety check on the L2 norm of the FP32 residual.
 *     [Novel Contributions, "Novel: Per-Iteration Safety Check"]
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers to memory the caller allocated
 *     and owns; the library never allocates, frees or retains them, and keeps
 *     no state between calls.
 *   - Work is enqueued asynchronously on `stream` (NULL = legacy default stream);
 *     a return of TL_OK means "validated and launched", not "finished".
 *   - Kernels are launched with programmatic dependent launch: one may be
 *     scheduled while the kernel before it on the stream is still finishing, but
 *     it touches no memory until that kernel has completed, so stream order holds
 *     exactly as for ordinary launches (inputs written by the preceding kernel are
 *     seen, outputs are not written before it is done).
 *   - Arguments are validated on the host before anything is launched; a
 *     non-TL_OK return means nothing was enqueued, except TL_ERR_CUDA, which
 *     reports a failed launch.  tl_last_error_message() gives details.
 *   - fp16 data are IEEE binary16 passed as `const void*`; weights are fp16
 *     row-major [out = d_model][in = d_model] (K = W_k h means
 *     K[r] = sum_c W_k[r][c] h[c]); head j owns rows j*head_dim .. (j+1)*head_dim-1.
 *   - Per-lane values read from device arrays (loops, ctx_len, start_pos) are
 *     range-checked on the device: an out-of-range lane is skipped (no output
 *     written, flags untouched) and TL_ERR_DEVICE_RANGE is recorded in the
 *     workspace status word (see tl_storeh_poll_status).  Device kernels never
 *     trap; every wait inside a kernel is bounded and records
 *     TL_ERR_DEVICE_TIMEOUT instead of hanging.
 */
#ifndef TL_STOREH_H
#define TL_STOREH_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TL_STOREH_ABI_VERSION 1

#if defined(__GNUC__)
#define TL_API __attribute__((visibility("default")))
#else
#define TL_API
#endif

/* Same type as cudaStream_t (CUDA runtime) and CUstream (driver API). */
typedef struct CUstream_st* tl_stream_t;

typedef enum {
  TL_OK = 0,
  TL_ERR_INVALID_ARG = 1,    /* NULL pointer, negative count, bad enum value */
  TL_ERR_SHAPE = 2,          /* d_model != n_heads * head_dim, or a size that breaks a layout rule */
  TL_ERR_CAPACITY = 3,       /* n_lanes > max_lanes, layer/iter outside the cache, workspace too small */
  TL_ERR_UNSUPPORTED = 4,    /* a shape the kernels are not built for (see tl_storeh_desc) */
  TL_ERR_CUDA = 5,           /* a CUDA runtime call or launch failed */
  TL_ERR_DEVICE_TIMEOUT = 6, /* a bounded wait inside a kernel gave up (recorded on the device) */
  TL_ERR_DEVICE_RANGE = 7    /* a per-lane device value was out of range; that lane was skipped */
} tl_status;

/* How a cached h row is stored. */
typedef enum {
  TL_H_FP16 = 0,       /* d fp16 values: 2*d bytes, no scale */
  TL_H_INT8_TOKEN = 1, /* d int8 codes + one fp32 scale per row:
                          scale = amax/127 (fp32 IEEE division),
                          code = clamp(rne(x / scale), -127, 127) */
  TL_H_INT4_G64 = 2    /* d/2 bytes of int4 codes + one fp16 scale per group of 64 along d:
                          scale = fp16_rne(amax_g / 7.0f),
                          code = clamp(rne(x / (float)scale), -7, 7);
                          byte j of a group = (code[2j] & 0xF) | (code[2j+1] & 0xF) << 4 */
} tl_h_format;

/*
 * Shape of one store-h cache.  Supported: head_dim in {64, 128};
 * d_model = n_heads * head_dim with d_model a multiple of 256 and at most 2048;
 * n_heads <= 16; 1 <= max_ctx <= 65536 counts every position including the newest token.
 * Precision of the decode: within max-abs 2e-3 and relative L2 1e-3 of an FP64 reference for
 * d_model <= 1024 in every format, and for d_model > 1024 where the outputs stay of order one
 * (INT4 rows, FP16 rows of unit scale).  Above d_model 1024 the absorbed query and the softmax
 * weights enter the tensor cores as single fp16 operands (their fp16 hi + lo parts do not fit
 * shared memory and tensor memory there), so outputs of large magnitude -- INT8 rows with
 * outlier rows 8x the rest reach |out| of about 25 -- stay within relative L2 1e-3 but can
 * exceed max-abs 2e-3 (3e-2 measured at d_model 1792).
 */
typedef struct {
  int32_t d_model;
  int32_t n_heads;
  int32_t head_dim;
  int32_t n_pre;     /* unique layers before the loop block */
  int32_t L_max;     /* loop iterations the cache is sized for */
  int32_t max_lanes; /* batch lanes the cache is sized for */
  int32_t max_ctx;   /* positions per (layer, lane) */
  int32_t fmt;       /* tl_h_format */
} tl_storeh_desc;

/*
 * Device memory of one cache, allocated by the caller with the sizes from
 * tl_storeh_cache_bytes.  Layout, row-major:
 *   codes [n_pre + L_max][max_lanes][max_ctx][row_code_bytes]
 *   scales[n_pre + L_max][max_lanes][max_ctx][row_scales]   (NULL for TL_H_FP16)
 * row_code_bytes = 2d (FP16), d (INT8), d/2 (INT4);
 * row_scales = 0 (FP16), 1 fp32 (INT8), d/64 fp16 (INT4).
 * Both base addresses must be 256-byte aligned.
 */
typedef struct {
  void* codes;
  void* scales;
} tl_storeh_cache;

/* Bytes the caller must allocate for the cache described by `desc`: the variable-L cache
 * holds n_pre + L_max layers [Architecture-Exclusive Features, "Variable-L KV cache"] of
 * max_lanes x max_ctx rows, each row stored in its mode's size [Architecture-Exclusive
 * Features, "Store-h KV cache", mode table: D (FP16-h), D/2 + e (INT8-h), D/4 + e (INT4-h)
 * per K+V pair of fp16 elements; here 2d, d + 4 and d/2 + 2 d/64 bytes, scales in
 * scales_bytes], laid out as tl_storeh_cache describes.
 * Errors: TL_ERR_INVALID_ARG (NULL), TL_ERR_SHAPE / TL_ERR_UNSUPPORTED (desc).
 * tl_storeh_desc.fmt is an int32_t holding a tl_h_format value rather than the enum type,
 * so that the struct's size and layout do not depend on the compiler's enum width. */
TL_API tl_status tl_storeh_cache_bytes(const tl_storeh_desc* desc, size_t* codes_bytes, size_t* scales_bytes);

/* Bytes of device workspace tl_storeh_attn_decode needs for up to `n_lanes`
 * lanes (256-byte aligned, contents need no initialisation apart from the status
 * word described at tl_storeh_poll_status, must not be shared by two calls in flight
 * at once).  It holds, per lane, the absorbed query q_j^T W_k[j] of every head and the
 * partial softmax results (running max, sum and sum_c p_c h_c) of each 1024-row split
 * of the lane's context: the absorbed form of the pages' K = W_k h rebuild
 * [Novel Contributions, "Novel Mechanism: Store-h KV Cache"], split so that the
 * context of one lane streams on several SMs at once.  One decode call takes at most
 * 64 lanes (TL_ERR_UNSUPPORTED above); larger batches are split into several calls. */
TL_API tl_status tl_storeh_workspace_bytes(const tl_storeh_desc* desc, int32_t n_lanes, size_t* bytes);

/*
 * Quantise fp16 h rows and write them into cache layer `layer`
 * [Architecture-Exclusive Features, "Store-h KV cache" — the write side;
 *  "Variable-L KV cache" — layer n_pre+i is filled by loop iteration i].
 *
 *   h_rows     device fp16 [n_lanes][n_rows][d_model]
 *   start_pos  device int32 [n_lanes]: row r of lane b goes to position start_pos[b] + r
 *   row_count  device int32 [n_lanes] or NULL: lane b writes rows r < row_count[b]
 *              (NULL: all n_rows)
 *   loops      device int32 [n_lanes] or NULL: lane b is skipped when
 *              layer >= n_pre + loops[b] (NULL: no lane is skipped)
 * Cache lane index = b.  Rows whose position falls outside [0, max_ctx) are not
 * written.  Codes and scales are bit-exact with the definitions in tl_h_format.
 * Errors: TL_ERR_INVALID_ARG, TL_ERR_CAPACITY (n_lanes > max_lanes, layer outside
 * [0, n_pre + L_max)), TL_ERR_SHAPE, TL_ERR_UNSUPPORTED, TL_ERR_CUDA.
 */
TL_API tl_status tl_storeh_append(const tl_storeh_desc* desc, tl_storeh_cache cache, int32_t layer,
                           const void* h_rows, int32_t n_lanes, int32_t n_rows,
                           const int32_t* start_pos, const int32_t* row_count,
                           const int32_t* loops, tl_stream_t stream);

/*
 * One loop iteration `iter` of store-h decode attention for a batch of lanes
 * [Novel Contributions, "Novel Mechanism: Store-h KV Cache"; Architecture-
 * Exclusive Features, "Store-h KV cache", "Variable-L KV cache", "L-aware
 * batching"].  For every lane b with iter < loops[b]:
 *   rows c = 0 .. ctx_len[b] of cache layer n_pre + iter are dequantised
 *   (row ctx_len[b] is the new token, already appended by tl_storeh_append);
 *   q = W_q h_new[b]; K_c = W_k h_c; V_c = W_v h_c; per head j:
 *   s_c = q_j . K_cj / sqrt(head_dim), p = softmax(s), out[b][j] = sum_c p_c V_cj.
 * The kernels use the algebraically equal absorbed form (q_j^T W_k[j] applied
 * to h, then W_v[j] applied to sum_c p_c h_c).  Lanes with iter >= loops[b]
 * are left untouched (their out rows are not written).
 *
 *   loops, ctx_len  device int32 [n_lanes]; 0 <= ctx_len[b] < max_ctx, loops[b] <= L_max
 *   h_new           device fp16 [n_lanes][d_model]: the new token's h (unquantised), for q
 *   W_q, W_k, W_v   device fp16 [d_model][d_model] (may be rows of one stacked [3d][d] buffer)
 *   out             device fp32 [n_lanes][n_heads][head_dim]
 *   residual        device fp32 [n_lanes][d_model] or NULL.  When given, the
 *                   per-iteration safety check of tl_residual_norm_check runs
 *                   in the same enqueue, with `threshold`, `abort_flags`,
 *                   `first_abort_iter` and `norms_out` as described there.
 *   workspace       device scratch of at least tl_storeh_workspace_bytes(desc, n_lanes)
 * Errors: TL_ERR_INVALID_ARG, TL_ERR_CAPACITY, TL_ERR_SHAPE, TL_ERR_UNSUPPORTED,
 * TL_ERR_CUDA; device-side conditions via tl_storeh_poll_status.
 */
TL_API tl_status tl_storeh_attn_decode(const tl_storeh_desc* desc, tl_storeh_cache cache, int32_t iter,
                                const int32_t* loops, const int32_t* ctx_len, const void* h_new,
                                const void* W_q, const void* W_k, const void* W_v, float* out,
                                const float* residual, float threshold, uint8_t* abort_flags,
                                int32_t* first_abort_iter, float* norms_out, void* workspace,
                                size_t workspace_bytes, int32_t n_lanes, tl_stream_t stream);

/*
 * tl_storeh_append followed by tl_storeh_attn_decode in one enqueue: for every lane b
 * with iter < loops[b] (and loops[b], ctx_len[b] in range), h_new[b] is first
 * quantised into cache layer n_pre + iter at position ctx_len[b] -- exactly what
 * tl_storeh_append(desc, cache, n_pre + iter, h_new, n_lanes, 1, ctx_len, NULL,
 * loops, stream) writes -- and then the decode of tl_storeh_attn_decode runs on it.
 * The append is done inside the decode's first kernel while its weight tiles load,
 * which saves a launch and its latency per iteration.  Arguments, results and
 * errors as for tl_storeh_attn_decode; h_new is both the row appended and the query
 * input.
 */
TL_API tl_status tl_storeh_append_attn_decode(const tl_storeh_desc* desc, tl_storeh_cache cache, int32_t iter,
                                const int32_t* loops, const int32_t* ctx_len, const void* h_new,
                                const void* W_q, const void* W_k, const void* W_v, float* out,
                                const float* residual, float threshold, uint8_t* abort_flags,
                                int32_t* first_abort_iter, float* norms_out, void* workspace,
                                size_t workspace_bytes, int32_t n_lanes, tl_stream_t stream);

/*
 * Tree verification over the store-h cache: many query tokens per lane in one enqueue
 * [Architecture-Exclusive Features, "Tree speculative decoding": K draft branches, each a
 * chain of D tokens grown from the same root, are verified in one mask-gated pass].
 * For every lane b with iter < loops[b]:
 *   1. the K x D tree tokens' h rows are quantised into cache layer n_pre + iter at positions
 *      ctx_len[b] + k*D + t (branch k, depth t), exactly as tl_storeh_append writes them;
 *   2. token (k, t) attends the lane's cached positions 0 .. ctx_len[b]-1 and its own
 *      branch's tokens (k, 0 .. t) -- itself included, no other branch -- with its query
 *      q = W_q h_tree[b][k][t] from the unquantised row, K = W_k h, V = W_v h and the softmax
 *      scale 1/sqrt(head_dim) of tl_storeh_attn_decode:
 *        out[b][k][t] = sum over those rows c of softmax(s)_c V_c.
 *   With one branch the pass equals `depth` sequential single-token decodes; token (0, t)
 *   reads exactly the rows (and in the same order) of a decode with ctx_len[b] + t cached
 *   positions, so its output is bit-identical to that decode's.
 *
 *   loops, ctx_len  device int32 [n_lanes]; ctx_len[b] + n_branches*depth <= max_ctx, or the
 *                   lane is skipped and TL_ERR_DEVICE_RANGE recorded (its tree rows that fit
 *                   are still written)
 *   h_tree          device fp16 [n_lanes][n_branches][depth][d_model]
 *   W_q, W_k, W_v   device fp16 [d_model][d_model]
 *   out             device fp32 [n_lanes][n_branches][depth][n_heads][head_dim]; rows of
 *                   inactive lanes are not written
 *   workspace       tl_storeh_verify_workspace_bytes(desc, n_lanes, n_branches, depth) bytes,
 *                   256-byte aligned, its first 256 bytes (the status word, read with
 *                   tl_storeh_poll_status) zeroed once
 * No safety check runs here (a verification pass has no residual of its own).
 * Supported: 1 <= n_branches * depth <= 1024.  The n_lanes * n_branches * depth query tokens
 * run in groups of 64 through the decode kernels, each token as a lane of its own.
 * Errors: TL_ERR_INVALID_ARG, TL_ERR_CAPACITY (n_lanes > max_lanes, iter outside [0, L_max),
 * workspace too small, a tree larger than max_ctx), TL_ERR_UNSUPPORTED, TL_ERR_CUDA.
 */
TL_API tl_status tl_storeh_verify_attn(const tl_storeh_desc* desc, tl_storeh_cache cache, int32_t iter,
                                       const int32_t* loops, const int32_t* ctx_len, const void* h_tree,
                                       int32_t n_branches, int32_t depth, const void* W_q, const void* W_k,
                                       const void* W_v, float* out, void* workspace, size_t workspace_bytes,
                                       int32_t n_lanes, tl_stream_t stream);

/* Workspace bytes of tl_storeh_verify_attn / tl_storeh_prefill_attn (prefill: n_branches = 1,
 * depth = n_tokens): a decode workspace for 64 query tokens (with one split more per token,
 * for its branch rows) plus 24 bytes per query token for its row map.
 * Errors: the desc errors, TL_ERR_INVALID_ARG, TL_ERR_CAPACITY, TL_ERR_UNSUPPORTED. */
TL_API tl_status tl_storeh_verify_workspace_bytes(const tl_storeh_desc* desc, int32_t n_lanes, int32_t n_branches,
                                                  int32_t depth, size_t* bytes);

/*
 * Chunked prefill over the store-h cache [Architecture-Exclusive Features, "What this list is
 * not": chunked prefill runs on the same cache; "Variable-L KV cache": loop iteration i fills
 * layer n_pre + i]: n_tokens new tokens per lane are appended at positions ctx_len[b] ..
 * ctx_len[b] + n_tokens - 1 of layer n_pre + iter and attend causally: token t attends
 * positions 0 .. ctx_len[b] + t.  This is tl_storeh_verify_attn with one branch of depth
 * n_tokens (same arguments, h_chunk [n_lanes][n_tokens][d_model], out
 * [n_lanes][n_tokens][n_heads][head_dim]); each token's output is bit-identical to the decode
 * of that token with ctx_len[b] + t cached positions.
 */
TL_API tl_status tl_storeh_prefill_attn(const tl_storeh_desc* desc, tl_storeh_cache cache, int32_t iter,
                                        const int32_t* loops, const int32_t* ctx_len, const void* h_chunk,
                                        int32_t n_tokens, const void* W_q, const void* W_k, const void* W_v,
                                        float* out, void* workspace, size_t workspace_bytes, int32_t n_lanes,
                                        tl_stream_t stream);

/*
 * Options of tl_storeh_decode_ex.  Zero-initialise the struct, then set what is needed.
 *   append      0: the decode of tl_storeh_attn_decode; 1: tl_storeh_append_attn_decode
 *               (h_new appended as the new token's row first).
 *   split_rows  context rows per split: 0 (the default, 1024) or one of 128, 256, 512, 1024.
 *               Each lane's context is cut into splits of this many rows, each streamed by
 *               its own CTA and merged exactly at the end.  A lane's result depends only on
 *               its own rows and on split_rows, never on the other lanes of the call
 *               [Architecture-Exclusive Features, "L-aware batching": mixed lanes give the
 *               bits of solo runs], so runs that are compared must use the same value.
 *               Shorter splits put more SMs on a lane, which pays when the call has few
 *               lanes or few active lanes (single-sequence decode, the deep iterations of
 *               an L-aware batch); they write more partial results (16 x d_model fp32 per
 *               split).  TL_ERR_UNSUPPORTED when the splits of max_ctx rows for n_lanes
 *               lanes would not fit the merge kernel's shared memory.
 *   reserved    must be zero.
 */
typedef struct {
  int32_t append;
  int32_t split_rows;
  int32_t reserved[7];
} tl_decode_opts;

/* tl_storeh_workspace_bytes for a call made with these options (NULL = defaults). */
TL_API tl_status tl_storeh_workspace_bytes_ex(const tl_storeh_desc* desc, int32_t n_lanes, const tl_decode_opts* opts,
                                              size_t* bytes);

/* tl_storeh_attn_decode / tl_storeh_append_attn_decode with options (see tl_decode_opts);
 * same arguments, results and errors, the workspace sized by tl_storeh_workspace_bytes_ex
 * with the same options.  TL_ERR_INVALID_ARG for a bad option. */
TL_API tl_status tl_storeh_decode_ex(const tl_storeh_desc* desc, tl_storeh_cache cache, int32_t iter,
                                     const int32_t* loops, const int32_t* ctx_len, const void* h_new,
                                     const void* W_q, const void* W_k, const void* W_v, float* out,
                                     const float* residual, float threshold, uint8_t* abort_flags,
                                     int32_t* first_abort_iter, float* norms_out, void* workspace,
                                     size_t workspace_bytes, int32_t n_lanes, const tl_decode_opts* opts,
                                     tl_stream_t stream);

/*
 * RoPE-compatible variant of tl_storeh_attn_decode, for models that put rotary position
 * embeddings on q and K.  The pages give K = W_k h with no positional encoding [Novel
 * Contributions, "Novel Mechanism: Store-h KV Cache"]; a rotation between the rebuild and the
 * score breaks the absorbed form for K, so this call rebuilds K = W_k h explicitly for every
 * attended row (a dense contraction, on the tensor cores) and rotates it.  Per head j:
 *   q' = R(ctx_len[b]) q_j,  K'_c = R(c) K_cj,  s_c = q' . K'_c / sqrt(head_dim),
 *   out[b][j] = sum_c softmax(s)_c V_cj   (V = W_v h, not rotated),
 * where R(t) rotates the pairs (i, i + head_dim/2), i < head_dim/2, by the angle
 * t * rope_base^(-2i/head_dim) (the "rotate half" form of rotary embeddings): row c of the
 * cache sits at position c and the new token's query at its own row, ctx_len[b].
 * Arguments, results and errors as tl_storeh_attn_decode (the new row already appended), plus
 *   rope_base  the rotary base (10000 in most models), > 1;
 *   workspace  tl_storeh_rope_workspace_bytes(desc, n_lanes) bytes, 256-byte aligned, its first
 *              256 bytes (the status word) zeroed once.
 * The explicit rebuild costs 2 d_model^2 FLOPs per attended row, head_dim times the absorbed
 * decode's; this call is compute-bound where tl_storeh_attn_decode is memory-bound.
 */
TL_API tl_status tl_storeh_attn_decode_rope(const tl_storeh_desc* desc, tl_storeh_cache cache, int32_t iter,
                                            const int32_t* loops, const int32_t* ctx_len, const void* h_new,
                                            const void* W_q, const void* W_k, const void* W_v, float* out,
                                            const float* residual, float threshold, uint8_t* abort_flags,
                                            int32_t* first_abort_iter, float* norms_out, float rope_base,
                                            void* workspace, size_t workspace_bytes, int32_t n_lanes,
                                            tl_stream_t stream);

/* Workspace bytes of tl_storeh_attn_decode_rope: the decode workspace plus the cos / sin table
 * of the cache's positions, the rotated queries and the scores (64 bytes per position and lane).
 * Errors: as tl_storeh_workspace_bytes. */
TL_API tl_status tl_storeh_rope_workspace_bytes(const tl_storeh_desc* desc, int32_t n_lanes, size_t* bytes);

/*
 * Per-iteration safety check [Novel Contributions, "Novel: Per-Iteration
 * Safety Check"; Architecture-Exclusive Features, "Per-iteration safety check"].
 * For every lane b with iter < loops[b] (all lanes when loops is NULL):
 *   n2 = sum_k residual[b][k]^2 accumulated in FP64 (each term exact);
 *   if n2 > threshold^2 (strict): abort_flags[b] = 1 and, if the flag was 0,
 *   first_abort_iter[b] = iter.  Flags are sticky (never cleared here).
 *   norms_out[b] = sqrt(n2) as fp32 when norms_out is not NULL.
 * Lanes with iter >= loops[b] are left untouched.
 *   residual          device fp32 [n_lanes][d]
 *   abort_flags       device uint8 [n_lanes], caller-initialised (0 = running)
 *   first_abort_iter  device int32 [n_lanes], caller-initialised (e.g. -1)
 * Errors: TL_ERR_INVALID_ARG, TL_ERR_CUDA.
 */
TL_API tl_status tl_residual_norm_check(const float* residual, int32_t n_lanes, int32_t d, float threshold,
                                 int32_t iter, const int32_t* loops, uint8_t* abort_flags,
                                 int32_t* first_abort_iter, float* norms_out, tl_stream_t stream);

/*
 * tl_storeh_attn_decode without a caller-supplied workspace, for callers that
 * cannot allocate device memory (no cudaMalloc, no allocator of their own:
 * plug-ins running inside a host application's memory budget, code that must
 * not allocate once a stream or graph is set up, and similar).  The pages have
 * no counterpart; this is a packaging variant of the decode above.
 *
 * Same arguments, meaning and results as tl_storeh_attn_decode, minus
 * `workspace` / `workspace_bytes`.  The scratch is a 32 MiB array compiled into
 * the library (a static __device__ variable): every GPU that loads the library
 * holds those 32 MiB until the process exits.  Requests whose workspace
 * (tl_storeh_workspace_bytes) would exceed 32 MiB are rejected with
 * TL_ERR_CAPACITY before anything is launched.  The call allocates nothing: no
 * cudaMalloc, cudaFree or allocating library routine.
 *
 * Every call looks up the array's device address (cudaGetSymbolAddress) in the
 * device and context current at the call.  Under CUDA's default lazy module
 * loading the array itself is created by the first such lookup on a device, so
 * the first call on each device is where the 32 MiB are taken and where an
 * out-of-memory condition shows up (TL_ERR_CUDA): make one warm-up call during
 * initialisation, and make it before any stream capture.  All calls in the
 * process share the one array and it
 * keeps the previous call's contents (the call clears the part that must start
 * at zero itself): two calls that may overlap on the GPU — on different streams
 * without an ordering between them — race on it and give wrong results.
 *   status_out  device uint32 or NULL: receives this call's device status word
 *               (bit 0 = a lane's loops/ctx_len was out of range and the lane was
 *               skipped, bit 1 = a bounded device wait gave up).  The word lives in
 *               the built-in array, which the next call clears and which
 *               tl_storeh_poll_status cannot reach: with status_out == NULL the
 *               range and timeout reports of this call are discarded.
 */
TL_API tl_status tl_storeh_attn_decode_static_ws(const tl_storeh_desc* desc, tl_storeh_cache cache, int32_t iter,
                                                 const int32_t* loops, const int32_t* ctx_len, const void* h_new,
                                                 const void* W_q, const void* W_k, const void* W_v, float* out,
                                                 const float* residual, float threshold, uint8_t* abort_flags,
                                                 int32_t* first_abort_iter, float* norms_out, int32_t n_lanes,
                                                 uint32_t* status_out, tl_stream_t stream);

/*
 * Synchronises `stream`, then reads and clears the status word that kernels
 * of tl_storeh_attn_decode record in `workspace`.  Returns TL_OK,
 * TL_ERR_DEVICE_TIMEOUT (a bounded device wait gave up), TL_ERR_DEVICE_RANGE
 * (a lane's loops/ctx_len was out of range and the lane was skipped) or
 * TL_ERR_CUDA.  The status word starts at the beginning of the workspace,
 * whose first 256 bytes are reserved for it; a freshly allocated workspace
 * must have those 256 bytes zero-filled once (or be cleared with this call)
 * before its first use.  When the word is not zero this call clears all 256
 * bytes.
 */
TL_API tl_status tl_storeh_poll_status(void* workspace, size_t workspace_bytes, tl_stream_t stream);

/*
 * Self-test of the device failure-detection path: enqueues one kernel whose only wait
 * can never complete (an mbarrier nothing arrives at), bounded by the helper every
 * kernel of the library uses.  After `limit_cycles` SM clocks it gives up and records
 * TL_ERR_DEVICE_TIMEOUT in the workspace status word, as a kernel that timed out in
 * earnest would; tl_storeh_poll_status then returns it and clears the word.  No GPU
 * fault, trap or hang is involved, and the context stays usable.
 *   workspace     a decode workspace (only its status word is touched)
 *   limit_cycles  in (0, 4e9] SM clocks
 * Errors: TL_ERR_INVALID_ARG, TL_ERR_CUDA.
 */
TL_API tl_status tl_storeh_selftest_wait_timeout(void* workspace, size_t workspace_bytes, int64_t limit_cycles,
                                                 tl_stream_t stream);

/*
 * Measurement hook (optional).  While a tl_profile is installed on the calling
 * thread, every tl_storeh_* call made from that thread counts the kernels it
 * launches in `launches`, and records begin_events[k] / end_events[k]
 * (cudaEvent_t handles created by the caller) on the call's stream right before
 * and right after each launch of the call's dominant kernel -- the context-streaming
 * kernel of the decode, verification, prefill and delta calls, the score kernel (the
 * K rebuild) of tl_storeh_attn_decode_rope -- for k = recorded++ while recorded < capacity.
 * Pass NULL to uninstall.  The struct must outlive its installation.  The events
 * sit between kernels, which stops a kernel from being scheduled during the tail
 * of the one before it, so a step timed with the hook installed runs a little
 * slower than one without.
 */
typedef struct {
  void** begin_events;
  void** end_events;
  int32_t capacity;
  int32_t recorded;
  int64_t launches;
} tl_profile;

TL_API tl_status tl_set_profile(tl_profile* profile);

/* Static description of a status code. */
TL_API const char* tl_status_string(tl_status status);

/* Details of the most recent non-TL_OK return on the calling thread. */
TL_API const char* tl_last_error_message(void);

/* TL_STOREH_ABI_VERSION of the loaded library. */
TL_API int32_t tl_storeh_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TL_STOREH_H */
