// C ABI of the RoPE-compatible decode (include/tl_storeh.h, tl_storeh_attn_decode_rope).
#include "tl_internal.cuh"

namespace tl {
namespace {

struct RopeWorkspace {
  Workspace wl;  // the decode workspace (status word, split partials)
  size_t cs_off, qrot_off, scores_off, total;
};

RopeWorkspace rope_workspace(const Shape& s, int n_lanes) {
  RopeWorkspace w;
  w.wl = workspace_layout(s, n_lanes);
  w.cs_off = align256(w.wl.total);
  w.qrot_off = w.cs_off + align256((size_t)s.max_ctx * (s.hd / 2) * sizeof(float2));
  w.scores_off = w.qrot_off + align256((size_t)n_lanes * s.d * 4);
  w.total = w.scores_off + align256((size_t)n_lanes * s.max_ctx * kMaxHeads * 4);
  return w;
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

tl_status rope_shape(const tl_storeh_desc* desc, int32_t n_lanes, Shape* s) {
  size_t cb, sb, wb;
  tl_status st = tl_storeh_cache_bytes(desc, &cb, &sb);
  if (st != TL_OK) return st;
  if ((st = tl_storeh_workspace_bytes(desc, n_lanes, &wb)) != TL_OK) return st;
  *s = Shape{desc->d_model, desc->n_heads, desc->head_dim, desc->n_pre, desc->L_max, desc->max_lanes, desc->max_ctx,
             desc->fmt};
  return TL_OK;
}

}  // namespace
}  // namespace tl

extern "C" {

tl_status tl_storeh_rope_workspace_bytes(const tl_storeh_desc* desc, int32_t n_lanes, size_t* bytes) {
  tl::Shape s{};
  tl_status st = tl::rope_shape(desc, n_lanes, &s);
  if (st != TL_OK) return st;
  if (!bytes) return tl::set_error(TL_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = tl::rope_workspace(s, n_lanes).total;
  return TL_OK;
}

tl_status tl_storeh_attn_decode_rope(const tl_storeh_desc* desc, tl_storeh_cache cache, int32_t iter,
                                     const int32_t* loops, const int32_t* ctx_len, const void* h_new,
                                     const void* W_q, const void* W_k, const void* W_v, float* out,
                                     const float* residual, float threshold, uint8_t* abort_flags,
                                     int32_t* first_abort_iter, float* norms_out, float rope_base, void* workspace,
                                     size_t workspace_bytes, int32_t n_lanes, tl_stream_t stream) {
  using namespace tl;
  Shape s{};
  tl_status st = rope_shape(desc, n_lanes, &s);
  if (st != TL_OK) return st;
  if (!cache.codes || (s.fmt != TL_H_FP16 && !cache.scales)) return set_error(TL_ERR_INVALID_ARG, "cache buffer is NULL");
  if (!aligned(cache.codes, 256) || (cache.scales && !aligned(cache.scales, 256)))
    return set_error(TL_ERR_INVALID_ARG, "cache buffers must be 256-byte aligned");
  if (!loops || !ctx_len || !h_new || !W_q || !W_k || !W_v || !out || !workspace)
    return set_error(TL_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned(h_new, 16) || !aligned(W_q, 16) || !aligned(W_k, 16) || !aligned(W_v, 16) || !aligned(out, 16))
    return set_error(TL_ERR_INVALID_ARG, "h_new, W_q, W_k, W_v and out must be 16-byte aligned");
  if (!aligned(workspace, 256)) return set_error(TL_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (iter < 0 || iter >= s.L_max) return set_error(TL_ERR_CAPACITY, "iter %d outside [0, L_max=%d)", iter, s.L_max);
  if (!(rope_base > 1.0f) || !(rope_base < 1e30f)) return set_error(TL_ERR_INVALID_ARG, "rope_base must be > 1 and finite");
  if (residual && (!abort_flags || !first_abort_iter))
    return set_error(TL_ERR_INVALID_ARG, "residual given without abort_flags / first_abort_iter");
  if (residual && !(threshold >= 0.0f)) return set_error(TL_ERR_INVALID_ARG, "threshold must be a non-negative number");
  const RopeWorkspace w = rope_workspace(s, n_lanes);
  if (workspace_bytes < w.total)
    return set_error(TL_ERR_CAPACITY, "workspace %zu bytes < %zu needed", workspace_bytes, w.total);
  uint8_t* ws = (uint8_t*)workspace;
  DecodeArgs a{s, cache.codes, cache.scales, iter, loops, ctx_len, (const __half*)h_new, (const __half*)W_q,
               (const __half*)W_k, (const __half*)W_v, out, n_lanes, ws, w.wl, residual, threshold, abort_flags,
               first_abort_iter, norms_out};
  a.scores = (const float*)(ws + w.scores_off);
  cudaStream_t cs = (cudaStream_t)stream;
  cudaError_t e = launch_rope_scores(a, rope_base, (float2*)(ws + w.cs_off), (float*)(ws + w.qrot_off),
                                     (float*)(ws + w.scores_off), cs);
  if (e == cudaSuccess) e = launch_stream(a, cs);
  if (e == cudaSuccess) e = launch_oproj(a, cs);
  if (e != cudaSuccess) return set_error(TL_ERR_CUDA, "rope decode launch: %s", cudaGetErrorString(e));
  return TL_OK;
}

}  // extern "C"
