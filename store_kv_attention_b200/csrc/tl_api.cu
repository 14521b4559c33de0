// C ABI of libtlstoreh.so: host-side validation and kernel launches.
// The operations are defined in include/tl_storeh.h.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "delta_internal.cuh"
#include "tl_delta.h"
#include "tl_internal.cuh"

namespace {

thread_local char g_msg[512] = "";

tl_status fail(tl_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof g_msg, fmt, ap);
  va_end(ap);
  return st;
}

tl_status cuda_fail(cudaError_t e, const char* what) {
  return fail(TL_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

// Validates a cache descriptor and converts it to the internal shape.
tl_status check_desc(const tl_storeh_desc* d, tl::Shape* s) {
  if (!d) return fail(TL_ERR_INVALID_ARG, "desc is NULL");
  if (d->fmt < TL_H_FP16 || d->fmt > TL_H_INT4_G64) return fail(TL_ERR_INVALID_ARG, "fmt %d is not a tl_h_format", d->fmt);
  if (d->d_model <= 0 || d->n_heads <= 0 || d->head_dim <= 0 || d->n_pre < 0 || d->L_max <= 0 ||
      d->max_lanes <= 0 || d->max_ctx <= 0)
    return fail(TL_ERR_INVALID_ARG, "desc has a non-positive size");
  if ((int64_t)d->n_heads * d->head_dim != d->d_model)
    return fail(TL_ERR_SHAPE, "d_model %d != n_heads %d * head_dim %d", d->d_model, d->n_heads, d->head_dim);
  if (d->head_dim != 64 && d->head_dim != 128) return fail(TL_ERR_UNSUPPORTED, "head_dim %d not in {64, 128}", d->head_dim);
  if (d->d_model % 256 != 0 || d->d_model > 2048)
    return fail(TL_ERR_UNSUPPORTED, "d_model %d must be a multiple of 256 and at most 2048", d->d_model);
  if (d->n_heads > tl::kMaxHeads) return fail(TL_ERR_UNSUPPORTED, "n_heads %d > %d", d->n_heads, tl::kMaxHeads);
  if (d->max_ctx > tl::kMaxCtx) return fail(TL_ERR_UNSUPPORTED, "max_ctx %d > %d", d->max_ctx, tl::kMaxCtx);
  if ((int64_t)(d->n_pre + d->L_max) * d->max_lanes * d->max_ctx > ((int64_t)1 << 40))
    return fail(TL_ERR_CAPACITY, "cache has too many rows");
  *s = tl::Shape{d->d_model, d->n_heads, d->head_dim, d->n_pre, d->L_max, d->max_lanes, d->max_ctx, d->fmt};
  return TL_OK;
}

// Validates a delta-cache descriptor (include/tl_delta.h).
tl_status check_delta_desc(const tl_delta_desc* d, tl::DeltaShape* s) {
  if (!d) return fail(TL_ERR_INVALID_ARG, "desc is NULL");
  if (d->d_model <= 0 || d->n_heads <= 0 || d->head_dim <= 0 || d->L_max <= 0 || d->max_lanes <= 0 ||
      d->max_ctx <= 0)
    return fail(TL_ERR_INVALID_ARG, "desc has a non-positive size");
  if ((int64_t)d->n_heads * d->head_dim != d->d_model)
    return fail(TL_ERR_SHAPE, "d_model %d != n_heads %d * head_dim %d", d->d_model, d->n_heads, d->head_dim);
  if (d->head_dim != 64 && d->head_dim != 128) return fail(TL_ERR_UNSUPPORTED, "head_dim %d not in {64, 128}", d->head_dim);
  if (d->d_model % 256 != 0 || d->d_model > 2048)
    return fail(TL_ERR_UNSUPPORTED, "d_model %d must be a multiple of 256 and at most 2048", d->d_model);
  if ((int64_t)d->L_max * d->max_lanes * d->max_ctx > ((int64_t)1 << 40))
    return fail(TL_ERR_CAPACITY, "cache has too many rows");
  *s = tl::DeltaShape{d->d_model, d->n_heads, d->head_dim, d->L_max, d->max_lanes, d->max_ctx};
  return TL_OK;
}

// A delta decode uses the store-h decode's projection kernels with the rows in natural d order
// (the FP16 layout): the shape they see (one loop iteration, the lane's 0/1 flag as its loop
// count) and the workspace layout [decode workspace | wloops | dloops].
tl::Shape delta_view_shape(const tl::DeltaShape& s, int n_lanes) {
  return tl::Shape{s.d, s.H, s.hd, 0, 1, n_lanes, s.max_ctx, TL_H_FP16};
}
struct DeltaWorkspace {
  tl::Workspace wl;
  size_t wloops_off, dloops_off, total;
};
DeltaWorkspace delta_workspace(const tl::DeltaShape& s, int n_lanes) {
  DeltaWorkspace w;
  // 256-row splits: this path's streaming kernel works through a split sequentially, so a lane
  // is spread over more SMs; the plan still depends on the lane's own context only
  w.wl = tl::workspace_layout(delta_view_shape(s, n_lanes), n_lanes, 0, tl::kDeltaSplitRows, /*qt_split=*/true);
  w.wloops_off = tl::align256(w.wl.total);
  w.dloops_off = w.wloops_off + tl::align256((size_t)n_lanes * 4);
  w.total = w.dloops_off + tl::align256((size_t)n_lanes * 4);
  return w;
}

tl_status check_cache(const tl::Shape& s, const tl_storeh_cache& c) {
  if (!c.codes) return fail(TL_ERR_INVALID_ARG, "cache.codes is NULL");
  if (s.fmt != TL_H_FP16 && !c.scales) return fail(TL_ERR_INVALID_ARG, "cache.scales is NULL");
  if (!aligned(c.codes, 256) || (c.scales && !aligned(c.scales, 256)))
    return fail(TL_ERR_INVALID_ARG, "cache buffers must be 256-byte aligned");
  return TL_OK;
}

}  // namespace

namespace tl {

tl_status set_error(tl_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof g_msg, fmt, ap);
  va_end(ap);
  return st;
}

tl_profile*& current_profile() {
  thread_local tl_profile* p = nullptr;
  return p;
}

void profile_stream_begin(cudaStream_t st) {
  tl_profile* p = current_profile();
  if (p && p->recorded < p->capacity) cudaEventRecord((cudaEvent_t)p->begin_events[p->recorded], st);
}

void profile_stream_end(cudaStream_t st) {
  tl_profile* p = current_profile();
  if (p && p->recorded < p->capacity) cudaEventRecord((cudaEvent_t)p->end_events[p->recorded++], st);
}

cudaError_t dyn_smem_limit(const void* func, int* limit) {
  struct Entry {
    const void* func;
    int dev, limit;
  };
  static std::mutex mu;
  static Entry table[64];
  static int n_entries = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n_entries; ++i)
      if (table[i].func == func && table[i].dev == dev) {
        *limit = table[i].limit;
        return cudaSuccess;
      }
  }
  cudaFuncAttributes fa;
  if ((e = cudaFuncGetAttributes(&fa, func)) != cudaSuccess) return e;
  int optin = 0;
  if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
  const int lim = optin - (int)fa.sharedSizeBytes;
  if ((e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, lim)) != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  if (n_entries < 64) table[n_entries++] = Entry{func, dev, lim};  // a full table only costs re-queries
  *limit = lim;
  return cudaSuccess;
}

}  // namespace tl

extern "C" {

tl_status tl_set_profile(tl_profile* profile) {
  if (profile && profile->capacity > 0 && (!profile->begin_events || !profile->end_events))
    return fail(TL_ERR_INVALID_ARG, "profile events are NULL");
  tl::current_profile() = profile;
  return TL_OK;
}

int32_t tl_storeh_abi_version(void) { return TL_STOREH_ABI_VERSION; }

const char* tl_last_error_message(void) { return g_msg; }

const char* tl_status_string(tl_status st) {
  switch (st) {
    case TL_OK: return "TL_OK";
    case TL_ERR_INVALID_ARG: return "TL_ERR_INVALID_ARG: a NULL pointer, negative count or bad enum value";
    case TL_ERR_SHAPE: return "TL_ERR_SHAPE: inconsistent sizes";
    case TL_ERR_CAPACITY: return "TL_ERR_CAPACITY: request exceeds the cache or workspace";
    case TL_ERR_UNSUPPORTED: return "TL_ERR_UNSUPPORTED: shape not supported by the kernels";
    case TL_ERR_CUDA: return "TL_ERR_CUDA: a CUDA call failed";
    case TL_ERR_DEVICE_TIMEOUT: return "TL_ERR_DEVICE_TIMEOUT: a bounded device wait gave up";
    case TL_ERR_DEVICE_RANGE: return "TL_ERR_DEVICE_RANGE: a per-lane device value was out of range";
  }
  return "unknown tl_status";
}

tl_status tl_storeh_cache_bytes(const tl_storeh_desc* desc, size_t* codes_bytes, size_t* scales_bytes) {
  tl::Shape s{};
  tl_status st = check_desc(desc, &s);
  if (st != TL_OK) return st;
  if (!codes_bytes || !scales_bytes) return fail(TL_ERR_INVALID_ARG, "output pointer is NULL");
  *codes_bytes = s.rows_total() * s.row_code_bytes();
  *scales_bytes = s.rows_total() * s.row_scales() * s.scale_bytes();
  return TL_OK;
}

// Split length of a call's options (0 = default); TL_OK or an error for a bad value or one whose
// merge state would not fit the epilogue kernel's shared memory.
static tl_status check_split(const tl::Shape& s, int32_t n_lanes, const tl_decode_opts* opts, int* split) {
  *split = tl::kSplitRows;
  if (opts && opts->split_rows != 0) {
    if (!tl::valid_split_rows(opts->split_rows))
      return fail(TL_ERR_INVALID_ARG, "split_rows %d not in {0, 128, 256, 512, 1024}", opts->split_rows);
    *split = opts->split_rows;
  }
  if (opts)
    for (int i = 0; i < 7; ++i)
      if (opts->reserved[i] != 0) return fail(TL_ERR_INVALID_ARG, "tl_decode_opts.reserved[%d] is not zero", i);
  const int s_max = tl::splits_for_rows(s.max_ctx, *split);
  if (tl::oproj_smem_bytes(s, n_lanes, s_max) > 227u * 1024u)
    return fail(TL_ERR_UNSUPPORTED, "split_rows %d: %d splits per lane for %d lanes exceed the merge kernel's shared memory",
                *split, s_max, n_lanes);
  return TL_OK;
}

static tl_status workspace_bytes_impl(const tl_storeh_desc* desc, int32_t n_lanes, const tl_decode_opts* opts,
                                      size_t* bytes) {
  tl::Shape s{};
  tl_status st = check_desc(desc, &s);
  if (st != TL_OK) return st;
  if (!bytes) return fail(TL_ERR_INVALID_ARG, "bytes is NULL");
  if (n_lanes <= 0) return fail(TL_ERR_INVALID_ARG, "n_lanes %d <= 0", n_lanes);
  if (n_lanes > s.max_lanes) return fail(TL_ERR_CAPACITY, "n_lanes %d > max_lanes %d", n_lanes, s.max_lanes);
  if (n_lanes > tl::kMaxGemmLanes)
    return fail(TL_ERR_UNSUPPORTED, "n_lanes %d > %d lanes per decode call", n_lanes, tl::kMaxGemmLanes);
  int split;
  if ((st = check_split(s, n_lanes, opts, &split)) != TL_OK) return st;
  *bytes = tl::workspace_layout(s, n_lanes, 0, split).total;
  return TL_OK;
}

tl_status tl_storeh_workspace_bytes(const tl_storeh_desc* desc, int32_t n_lanes, size_t* bytes) {
  return workspace_bytes_impl(desc, n_lanes, nullptr, bytes);
}

tl_status tl_storeh_workspace_bytes_ex(const tl_storeh_desc* desc, int32_t n_lanes, const tl_decode_opts* opts,
                                       size_t* bytes) {
  return workspace_bytes_impl(desc, n_lanes, opts, bytes);
}

tl_status tl_storeh_append(const tl_storeh_desc* desc, tl_storeh_cache cache, int32_t layer,
                           const void* h_rows, int32_t n_lanes, int32_t n_rows,
                           const int32_t* start_pos, const int32_t* row_count,
                           const int32_t* loops, tl_stream_t stream) {
  tl::Shape s{};
  tl_status st = check_desc(desc, &s);
  if (st != TL_OK) return st;
  if ((st = check_cache(s, cache)) != TL_OK) return st;
  if (!h_rows || !start_pos) return fail(TL_ERR_INVALID_ARG, "h_rows / start_pos is NULL");
  if (!aligned(h_rows, 16)) return fail(TL_ERR_INVALID_ARG, "h_rows must be 16-byte aligned");
  if (n_lanes <= 0 || n_rows < 0) return fail(TL_ERR_INVALID_ARG, "n_lanes %d / n_rows %d", n_lanes, n_rows);
  if (n_lanes > s.max_lanes) return fail(TL_ERR_CAPACITY, "n_lanes %d > max_lanes %d", n_lanes, s.max_lanes);
  if (layer < 0 || layer >= s.layers()) return fail(TL_ERR_CAPACITY, "layer %d outside [0, %d)", layer, s.layers());
  if (n_rows == 0) return TL_OK;
  cudaError_t e = tl::launch_append(s, cache.codes, cache.scales, layer, (const __half*)h_rows, n_lanes, n_rows,
                                    start_pos, row_count, loops, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "tl_storeh_append launch");
  return TL_OK;
}

tl_status tl_delta_cache_bytes(const tl_delta_desc* desc, size_t* anchor_bytes, size_t* delta_bytes,
                               size_t* scale_bytes) {
  tl::DeltaShape s{};
  tl_status st = check_delta_desc(desc, &s);
  if (st != TL_OK) return st;
  if (!anchor_bytes || !delta_bytes || !scale_bytes) return fail(TL_ERR_INVALID_ARG, "output pointer is NULL");
  const size_t rows = (size_t)s.max_lanes * s.max_ctx;
  *anchor_bytes = rows * s.d * 2;
  *delta_bytes = (size_t)(s.L_max - 1) * rows * s.d;
  *scale_bytes = (size_t)(s.L_max - 1) * rows * s.H * 2;
  return TL_OK;
}

tl_status tl_delta_append(const tl_delta_desc* desc, tl_delta_cache cache, int32_t iter, const void* h_rows,
                          int32_t n_lanes, int32_t n_rows, const int32_t* start_pos, const int32_t* loops,
                          tl_stream_t stream) {
  tl::DeltaShape s{};
  tl_status st = check_delta_desc(desc, &s);
  if (st != TL_OK) return st;
  if (!cache.anchor || (s.L_max > 1 && (!cache.deltas || !cache.scales)))
    return fail(TL_ERR_INVALID_ARG, "cache.anchor / deltas / scales is NULL");
  if (!aligned(cache.anchor, 256) || (cache.deltas && !aligned(cache.deltas, 256)) ||
      (cache.scales && !aligned(cache.scales, 256)))
    return fail(TL_ERR_INVALID_ARG, "cache buffers must be 256-byte aligned");
  if (!h_rows || !start_pos) return fail(TL_ERR_INVALID_ARG, "h_rows / start_pos is NULL");
  if (!aligned(h_rows, 16)) return fail(TL_ERR_INVALID_ARG, "h_rows must be 16-byte aligned");
  if (n_lanes <= 0 || n_rows < 0) return fail(TL_ERR_INVALID_ARG, "n_lanes %d / n_rows %d", n_lanes, n_rows);
  if (n_lanes > s.max_lanes) return fail(TL_ERR_CAPACITY, "n_lanes %d > max_lanes %d", n_lanes, s.max_lanes);
  if (iter < 0 || iter >= s.L_max) return fail(TL_ERR_CAPACITY, "iter %d outside [0, %d)", iter, s.L_max);
  if (n_rows == 0) return TL_OK;
  cudaError_t e = tl::launch_delta_append(s, cache.anchor, cache.deltas, cache.scales, iter, (const __half*)h_rows,
                                          n_lanes, n_rows, start_pos, loops, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "tl_delta_append launch");
  return TL_OK;
}

tl_status tl_delta_workspace_bytes(const tl_delta_desc* desc, int32_t n_lanes, size_t* bytes) {
  tl::DeltaShape s{};
  tl_status st = check_delta_desc(desc, &s);
  if (st != TL_OK) return st;
  if (!bytes) return fail(TL_ERR_INVALID_ARG, "bytes is NULL");
  if (n_lanes <= 0) return fail(TL_ERR_INVALID_ARG, "n_lanes %d <= 0", n_lanes);
  if (n_lanes > s.max_lanes) return fail(TL_ERR_CAPACITY, "n_lanes %d > max_lanes %d", n_lanes, s.max_lanes);
  if (n_lanes > tl::kMaxGemmLanes)
    return fail(TL_ERR_UNSUPPORTED, "n_lanes %d > %d lanes per decode call", n_lanes, tl::kMaxGemmLanes);
  if (s.H > tl::kMaxHeads) return fail(TL_ERR_UNSUPPORTED, "n_heads %d > %d", s.H, tl::kMaxHeads);
  if (s.max_ctx > tl::kMaxCtx) return fail(TL_ERR_UNSUPPORTED, "max_ctx %d > %d", s.max_ctx, tl::kMaxCtx);
  *bytes = delta_workspace(s, n_lanes).total;
  return TL_OK;
}

tl_status tl_delta_attn_decode(const tl_delta_desc* desc, tl_delta_cache cache, int32_t iter, const int32_t* loops,
                               const int32_t* ctx_len, const void* h_new, const void* W_q, const void* W_k,
                               const void* W_v, float* out, const float* residual, float threshold,
                               uint8_t* abort_flags, int32_t* first_abort_iter, float* norms_out, void* workspace,
                               size_t workspace_bytes, int32_t n_lanes, tl_stream_t stream) {
  tl::DeltaShape s{};
  tl_status st = check_delta_desc(desc, &s);
  if (st != TL_OK) return st;
  if (!cache.anchor || (s.L_max > 1 && (!cache.deltas || !cache.scales)))
    return fail(TL_ERR_INVALID_ARG, "cache.anchor / deltas / scales is NULL");
  if (!aligned(cache.anchor, 256) || (cache.deltas && !aligned(cache.deltas, 256)) ||
      (cache.scales && !aligned(cache.scales, 256)))
    return fail(TL_ERR_INVALID_ARG, "cache buffers must be 256-byte aligned");
  if (!loops || !ctx_len || !h_new || !W_q || !W_k || !W_v || !out || !workspace)
    return fail(TL_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned(h_new, 16) || !aligned(W_q, 16) || !aligned(W_k, 16) || !aligned(W_v, 16) || !aligned(out, 16))
    return fail(TL_ERR_INVALID_ARG, "h_new, W_q, W_k, W_v and out must be 16-byte aligned");
  if (!aligned(workspace, 256)) return fail(TL_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (n_lanes <= 0) return fail(TL_ERR_INVALID_ARG, "n_lanes %d <= 0", n_lanes);
  if (n_lanes > s.max_lanes) return fail(TL_ERR_CAPACITY, "n_lanes %d > max_lanes %d", n_lanes, s.max_lanes);
  if (iter < 0 || iter >= s.L_max) return fail(TL_ERR_CAPACITY, "iter %d outside [0, L_max=%d)", iter, s.L_max);
  if (n_lanes > tl::kMaxGemmLanes)
    return fail(TL_ERR_UNSUPPORTED, "n_lanes %d > %d lanes per decode call", n_lanes, tl::kMaxGemmLanes);
  if (s.H > tl::kMaxHeads) return fail(TL_ERR_UNSUPPORTED, "n_heads %d > %d", s.H, tl::kMaxHeads);
  if (s.max_ctx > tl::kMaxCtx) return fail(TL_ERR_UNSUPPORTED, "max_ctx %d > %d", s.max_ctx, tl::kMaxCtx);
  if (residual && (!abort_flags || !first_abort_iter))
    return fail(TL_ERR_INVALID_ARG, "residual given without abort_flags / first_abort_iter");
  if (residual && !(threshold >= 0.0f)) return fail(TL_ERR_INVALID_ARG, "threshold must be a non-negative number");
  const DeltaWorkspace w = delta_workspace(s, n_lanes);
  if (workspace_bytes < w.total) return fail(TL_ERR_CAPACITY, "workspace %zu bytes < %zu needed", workspace_bytes, w.total);

  uint8_t* ws = (uint8_t*)workspace;
  int32_t* wloops = (int32_t*)(ws + w.wloops_off);
  int32_t* dloops = (int32_t*)(ws + w.dloops_off);
  cudaStream_t cs = (cudaStream_t)stream;
  // 1. per-lane checks; 2. the new token's state of this iteration into the delta cache;
  // 3. q and the absorbed-query images; 4. the streaming stage, whose dequantisation is the FP32
  // prefix sum of the anchor and the deltas 1..iter; 5. the split merge and W_v; 6. the safety
  // check with the real iteration
  cudaError_t e = tl::launch_delta_prep(iter, s.L_max, s.max_ctx, n_lanes, loops, ctx_len, wloops, dloops,
                                        (uint32_t*)(ws + w.wl.status_off), cs);
  if (e == cudaSuccess)
    e = tl::launch_delta_append(s, cache.anchor, cache.deltas, cache.scales, iter, (const __half*)h_new, n_lanes, 1,
                                ctx_len, wloops, cs);
  if (e != cudaSuccess) return cuda_fail(e, "delta decode prologue launch");
  tl::DecodeArgs a{delta_view_shape(s, n_lanes), nullptr, nullptr, 0, dloops, ctx_len, (const __half*)h_new,
                   (const __half*)W_q, (const __half*)W_k, (const __half*)W_v, out, n_lanes, ws, w.wl,
                   nullptr, 0.0f, nullptr, nullptr, nullptr};
  e = tl::launch_qproj(a, cs);
  if (e == cudaSuccess) {
    tl::profile_stream_begin(cs);
    e = tl::launch_delta_stream(s, cache.anchor, cache.deltas, cache.scales, iter, n_lanes, dloops, ctx_len, ws, w.wl,
                                cs);
    tl::profile_stream_end(cs);
  }
  if (e == cudaSuccess) e = tl::launch_oproj(a, cs);
  if (e == cudaSuccess && residual)
    e = tl::launch_norm_check(residual, n_lanes, s.d, threshold, iter, wloops, abort_flags, first_abort_iter,
                              norms_out, cs);
  if (e != cudaSuccess) return cuda_fail(e, "delta decode launch");
  return TL_OK;
}

tl_status tl_residual_norm_check(const float* residual, int32_t n_lanes, int32_t d, float threshold,
                                 int32_t iter, const int32_t* loops, uint8_t* abort_flags,
                                 int32_t* first_abort_iter, float* norms_out, tl_stream_t stream) {
  if (!residual || !abort_flags || !first_abort_iter)
    return fail(TL_ERR_INVALID_ARG, "residual / abort_flags / first_abort_iter is NULL");
  if (n_lanes <= 0 || d <= 0 || iter < 0) return fail(TL_ERR_INVALID_ARG, "n_lanes %d, d %d, iter %d", n_lanes, d, iter);
  if (!(threshold >= 0.0f)) return fail(TL_ERR_INVALID_ARG, "threshold must be a non-negative number");
  cudaError_t e = tl::launch_norm_check(residual, n_lanes, d, threshold, iter, loops, abort_flags, first_abort_iter,
                                        norms_out, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "tl_residual_norm_check launch");
  return TL_OK;
}

namespace {
// The decode, optionally preceded (inside its first kernel) by the append of h_new as the new
// token's row of every active lane.
tl_status decode_impl(const tl_storeh_desc* desc, tl_storeh_cache cache, int32_t iter, const int32_t* loops,
                      const int32_t* ctx_len, const void* h_new, const void* W_q, const void* W_k, const void* W_v,
                      float* out, const float* residual, float threshold, uint8_t* abort_flags,
                      int32_t* first_abort_iter, float* norms_out, void* workspace, size_t workspace_bytes,
                      int32_t n_lanes, tl_stream_t stream, bool append, const tl_decode_opts* opts = nullptr) {
  tl::Shape s{};
  tl_status st = check_desc(desc, &s);
  if (st != TL_OK) return st;
  if ((st = check_cache(s, cache)) != TL_OK) return st;
  if (!loops || !ctx_len || !h_new || !W_q || !W_k || !W_v || !out || !workspace)
    return fail(TL_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned(h_new, 16) || !aligned(W_q, 16) || !aligned(W_k, 16) || !aligned(W_v, 16) || !aligned(out, 16))
    return fail(TL_ERR_INVALID_ARG, "h_new, W_q, W_k, W_v and out must be 16-byte aligned");
  if (!aligned(workspace, 256)) return fail(TL_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (n_lanes <= 0) return fail(TL_ERR_INVALID_ARG, "n_lanes %d <= 0", n_lanes);
  if (n_lanes > s.max_lanes) return fail(TL_ERR_CAPACITY, "n_lanes %d > max_lanes %d", n_lanes, s.max_lanes);
  if (iter < 0 || iter >= s.L_max) return fail(TL_ERR_CAPACITY, "iter %d outside [0, L_max=%d)", iter, s.L_max);
  if (n_lanes > tl::kMaxGemmLanes)
    return fail(TL_ERR_UNSUPPORTED, "n_lanes %d > %d lanes per decode call", n_lanes, tl::kMaxGemmLanes);
  if (residual && (!abort_flags || !first_abort_iter))
    return fail(TL_ERR_INVALID_ARG, "residual given without abort_flags / first_abort_iter");
  if (residual && !(threshold >= 0.0f)) return fail(TL_ERR_INVALID_ARG, "threshold must be a non-negative number");
  int split;
  if ((st = check_split(s, n_lanes, opts, &split)) != TL_OK) return st;
  tl::Workspace wl = tl::workspace_layout(s, n_lanes, 0, split);
  if (workspace_bytes < wl.total)
    return fail(TL_ERR_CAPACITY, "workspace %zu bytes < %zu needed", workspace_bytes, wl.total);

  tl::DecodeArgs a{s, cache.codes, cache.scales, iter, loops, ctx_len, (const __half*)h_new,
                   (const __half*)W_q, (const __half*)W_k, (const __half*)W_v, out, n_lanes,
                   (uint8_t*)workspace, wl, residual, threshold, abort_flags, first_abort_iter, norms_out};
  a.append = append;
  cudaStream_t cs = (cudaStream_t)stream;
  cudaError_t e = tl::launch_qproj(a, cs);
  if (e != cudaSuccess) return cuda_fail(e, "decode prologue launch");
  tl::profile_stream_begin(cs);
  e = tl::launch_stream(a, cs);
  tl::profile_stream_end(cs);
  if (e != cudaSuccess) return cuda_fail(e, "decode stream launch");
  e = tl::launch_oproj(a, cs);
  if (e != cudaSuccess) return cuda_fail(e, "decode epilogue launch");
  return TL_OK;
}
}  // namespace

tl_status tl_storeh_attn_decode(const tl_storeh_desc* desc, tl_storeh_cache cache, int32_t iter,
                                const int32_t* loops, const int32_t* ctx_len, const void* h_new,
                                const void* W_q, const void* W_k, const void* W_v, float* out,
                                const float* residual, float threshold, uint8_t* abort_flags,
                                int32_t* first_abort_iter, float* norms_out, void* workspace,
                                size_t workspace_bytes, int32_t n_lanes, tl_stream_t stream) {
  return decode_impl(desc, cache, iter, loops, ctx_len, h_new, W_q, W_k, W_v, out, residual, threshold, abort_flags, first_abort_iter, norms_out, workspace, workspace_bytes, n_lanes, stream, false);
}

tl_status tl_storeh_append_attn_decode(const tl_storeh_desc* desc, tl_storeh_cache cache, int32_t iter,
                                const int32_t* loops, const int32_t* ctx_len, const void* h_new,
                                const void* W_q, const void* W_k, const void* W_v, float* out,
                                const float* residual, float threshold, uint8_t* abort_flags,
                                int32_t* first_abort_iter, float* norms_out, void* workspace,
                                size_t workspace_bytes, int32_t n_lanes, tl_stream_t stream) {
  return decode_impl(desc, cache, iter, loops, ctx_len, h_new, W_q, W_k, W_v, out, residual, threshold, abort_flags, first_abort_iter, norms_out, workspace, workspace_bytes, n_lanes, stream, true);
}

tl_status tl_storeh_decode_ex(const tl_storeh_desc* desc, tl_storeh_cache cache, int32_t iter, const int32_t* loops,
                              const int32_t* ctx_len, const void* h_new, const void* W_q, const void* W_k,
                              const void* W_v, float* out, const float* residual, float threshold,
                              uint8_t* abort_flags, int32_t* first_abort_iter, float* norms_out, void* workspace,
                              size_t workspace_bytes, int32_t n_lanes, const tl_decode_opts* opts,
                              tl_stream_t stream) {
  if (!opts) return fail(TL_ERR_INVALID_ARG, "opts is NULL");
  if (opts->append != 0 && opts->append != 1) return fail(TL_ERR_INVALID_ARG, "opts->append %d not 0 or 1", opts->append);
  return decode_impl(desc, cache, iter, loops, ctx_len, h_new, W_q, W_k, W_v, out, residual, threshold, abort_flags,
                     first_abort_iter, norms_out, workspace, workspace_bytes, n_lanes, stream, opts->append == 1, opts);
}

tl_status tl_storeh_selftest_wait_timeout(void* workspace, size_t workspace_bytes, int64_t limit_cycles,
                                          tl_stream_t stream) {
  if (!workspace || workspace_bytes < 256) return fail(TL_ERR_INVALID_ARG, "workspace is NULL or too small");
  if (!aligned(workspace, 256)) return fail(TL_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (limit_cycles <= 0 || limit_cycles > (int64_t)4000000000ll)
    return fail(TL_ERR_INVALID_ARG, "limit_cycles %lld outside (0, 4e9]", (long long)limit_cycles);
  cudaError_t e = tl::launch_wait_selftest((uint32_t*)workspace, (long long)limit_cycles, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "tl_storeh_selftest_wait_timeout launch");
  return TL_OK;
}

tl_status tl_storeh_poll_status(void* workspace, size_t workspace_bytes, tl_stream_t stream) {
  if (!workspace || workspace_bytes < 256) return fail(TL_ERR_INVALID_ARG, "workspace is NULL or too small");
  cudaStream_t cs = (cudaStream_t)stream;
  uint32_t word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof word, cudaMemcpyDeviceToHost, cs);
  if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
  if (e != cudaSuccess) return cuda_fail(e, "reading the status word");
  if (word != 0) {
    e = cudaMemsetAsync(workspace, 0, 256, cs);  // the status block
    if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the status word");
  }
  if (word & tl::kStatusTimeout) return fail(TL_ERR_DEVICE_TIMEOUT, "device status word 0x%x", word);
  if (word & tl::kStatusRange) return fail(TL_ERR_DEVICE_RANGE, "device status word 0x%x", word);
  return TL_OK;
}

}  // extern "C"
