// Multi-query attention over the store-h cache: tree verification and chunked prefill.
// [Architecture-Exclusive Features, "Tree speculative decoding": K draft branches, each a chain
//  of D tokens grown from the same root, verified in one mask-gated pass; "What this list is
//  not": chunked prefill over the same cache]
//
// Every query token becomes a virtual lane of the decode kernels: token (b, k, t) has its own
// query (its unquantised h) and attends two contiguous runs of rows of its physical lane b:
// the cached positions [0, ctx_len[b]) and its own branch's tokens up to itself,
// [ctx_len[b] + k D, ctx_len[b] + k D + t].  The tree rows are appended first (the bulk
// append), so they are read back in the cache's format like a decode's new token.  For
// branch 0 the two runs touch and are merged, so a prefill chunk (one branch) attends one run
// [0, ctx_len[b] + t] per token, exactly the rows (and split plan) of a decode with
// ctx_len[b] + t cached positions.
#include "tl_internal.cuh"

namespace tl {
namespace {

// One thread per virtual lane v = (b * K + k) * D + t: its loop count and attended row count
// (the arrays the decode kernels take for loops / ctx_len) and its rows.  A lane whose loops /
// ctx_len are out of range, or whose tree does not fit the cache, is skipped and recorded.
__global__ void verify_prep_kernel(int n_virtual, int K, int D, int L_max, int max_ctx, const int32_t* loops,
                                   const int32_t* ctx_len, int32_t* vloops, int32_t* vctx, LaneSeg* seg,
                                   uint32_t* status) {
  const int v = blockIdx.x * blockDim.x + threadIdx.x;
  if (v >= n_virtual) return;
  const int b = v / (K * D), k = (v / D) % K, t = v % D;
  const int L = loops[b], c = ctx_len[b];
  const bool ok = L >= 0 && L <= L_max && c >= 0 && (long long)c + (long long)K * D <= max_ctx;
  if (!ok) {
    if (k == 0 && t == 0) atomicOr(status, kStatusRange);
    vloops[v] = 0;
    vctx[v] = 0;
    seg[v] = LaneSeg{b, 0, 0, 0};
    return;
  }
  LaneSeg g{b, c, c + k * D, t + 1};
  if (g.start1 == g.n0) {  // the runs touch: one run
    g.n0 += g.n1;
    g.n1 = 0;
  }
  vloops[v] = L;
  vctx[v] = g.n0 + g.n1 - 1;  // attended rows - 1: what a decode lane's ctx_len is
  seg[v] = g;
}

struct VerifyWorkspace {
  Workspace wl;  // decode workspace for one group of at most kMaxGemmLanes virtual lanes
  size_t vloops_off, vctx_off, seg_off, total;
  int group;
};

VerifyWorkspace verify_workspace(const Shape& s, int n_lanes, int K, int D) {
  VerifyWorkspace w;
  const int V = n_lanes * K * D;
  w.group = V < kMaxGemmLanes ? V : kMaxGemmLanes;
  w.wl = workspace_layout(s, w.group, 1);  // the branch run starts a split of its own
  w.vloops_off = align256(w.wl.total);
  w.vctx_off = w.vloops_off + align256((size_t)V * 4);
  w.seg_off = w.vctx_off + align256((size_t)V * 4);
  w.total = w.seg_off + align256((size_t)V * sizeof(LaneSeg));
  return w;
}

tl_status check_tree(const tl_storeh_desc* desc, int32_t n_lanes, int32_t K, int32_t D, Shape* s) {
  size_t cb, sb;
  tl_status st = tl_storeh_cache_bytes(desc, &cb, &sb);  // validates the descriptor
  if (st != TL_OK) return st;
  *s = Shape{desc->d_model, desc->n_heads, desc->head_dim, desc->n_pre, desc->L_max, desc->max_lanes,
             desc->max_ctx, desc->fmt};
  if (n_lanes <= 0 || K <= 0 || D <= 0)
    return set_error(TL_ERR_INVALID_ARG, "n_lanes %d, n_branches %d, depth %d must be positive", n_lanes, K, D);
  if (n_lanes > s->max_lanes) return set_error(TL_ERR_CAPACITY, "n_lanes %d > max_lanes %d", n_lanes, s->max_lanes);
  if ((long long)K * D > kSplitRows)
    return set_error(TL_ERR_UNSUPPORTED, "n_branches x depth = %lld > %d tree tokens per lane", (long long)K * D,
                     kSplitRows);
  if ((long long)K * D > s->max_ctx)
    return set_error(TL_ERR_CAPACITY, "n_branches x depth = %lld > max_ctx %d", (long long)K * D, s->max_ctx);
  if ((long long)n_lanes * K * D > (1 << 20))
    return set_error(TL_ERR_UNSUPPORTED, "more than 2^20 query tokens in one call");
  return TL_OK;
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

}  // namespace
}  // namespace tl

extern "C" {

tl_status tl_storeh_verify_workspace_bytes(const tl_storeh_desc* desc, int32_t n_lanes, int32_t n_branches,
                                           int32_t depth, size_t* bytes) {
  tl::Shape s{};
  tl_status st = tl::check_tree(desc, n_lanes, n_branches, depth, &s);
  if (st != TL_OK) return st;
  if (!bytes) return tl::set_error(TL_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = tl::verify_workspace(s, n_lanes, n_branches, depth).total;
  return TL_OK;
}

tl_status tl_storeh_verify_attn(const tl_storeh_desc* desc, tl_storeh_cache cache, int32_t iter,
                                const int32_t* loops, const int32_t* ctx_len, const void* h_tree, int32_t n_branches,
                                int32_t depth, const void* W_q, const void* W_k, const void* W_v, float* out,
                                void* workspace, size_t workspace_bytes, int32_t n_lanes, tl_stream_t stream) {
  using namespace tl;
  Shape s{};
  tl_status st = check_tree(desc, n_lanes, n_branches, depth, &s);
  if (st != TL_OK) return st;
  if (!cache.codes || (s.fmt != TL_H_FP16 && !cache.scales)) return set_error(TL_ERR_INVALID_ARG, "cache buffer is NULL");
  if (!aligned(cache.codes, 256) || (cache.scales && !aligned(cache.scales, 256)))
    return set_error(TL_ERR_INVALID_ARG, "cache buffers must be 256-byte aligned");
  if (!loops || !ctx_len || !h_tree || !W_q || !W_k || !W_v || !out || !workspace)
    return set_error(TL_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned(h_tree, 16) || !aligned(W_q, 16) || !aligned(W_k, 16) || !aligned(W_v, 16) || !aligned(out, 16))
    return set_error(TL_ERR_INVALID_ARG, "h_tree, W_q, W_k, W_v and out must be 16-byte aligned");
  if (!aligned(workspace, 256)) return set_error(TL_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if (iter < 0 || iter >= s.L_max) return set_error(TL_ERR_CAPACITY, "iter %d outside [0, L_max=%d)", iter, s.L_max);
  const int K = n_branches, D = depth, V = n_lanes * K * D;
  const VerifyWorkspace w = verify_workspace(s, n_lanes, K, D);
  if (workspace_bytes < w.total)
    return set_error(TL_ERR_CAPACITY, "workspace %zu bytes < %zu needed", workspace_bytes, w.total);

  uint8_t* ws = (uint8_t*)workspace;
  int32_t* vloops = (int32_t*)(ws + w.vloops_off);
  int32_t* vctx = (int32_t*)(ws + w.vctx_off);
  LaneSeg* seg = (LaneSeg*)(ws + w.seg_off);
  cudaStream_t cs = (cudaStream_t)stream;
  // 1. every query token's rows; 2. the tree rows into the cache at ctx_len[b] + k D + t
  verify_prep_kernel<<<(V + 127) / 128, 128, 0, cs>>>(V, K, D, s.L_max, s.max_ctx, loops, ctx_len, vloops, vctx, seg,
                                                      (uint32_t*)(ws + w.wl.status_off));
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess)
    e = launch_append(s, cache.codes, cache.scales, s.n_pre + iter, (const __half*)h_tree, n_lanes, K * D, ctx_len,
                      nullptr, loops, cs);
  if (e != cudaSuccess) return set_error(TL_ERR_CUDA, "verify prologue launch: %s", cudaGetErrorString(e));
  // 3. the decode kernels over groups of at most kMaxGemmLanes virtual lanes
  for (int g0 = 0; g0 < V; g0 += w.group) {
    const int G = V - g0 < w.group ? V - g0 : w.group;
    DecodeArgs a{s, cache.codes, cache.scales, iter, vloops + g0, vctx + g0,
                 (const __half*)h_tree + (size_t)g0 * s.d, (const __half*)W_q, (const __half*)W_k,
                 (const __half*)W_v, out + (size_t)g0 * s.d, G, ws, workspace_layout(s, G, 1),
                 nullptr, 0.0f, nullptr, nullptr, nullptr};
    a.seg = seg + g0;
    e = launch_qproj(a, cs);
    if (e == cudaSuccess) {
      profile_stream_begin(cs);
      e = launch_stream(a, cs);
      profile_stream_end(cs);
    }
    if (e == cudaSuccess) e = launch_oproj(a, cs);
    if (e != cudaSuccess) return set_error(TL_ERR_CUDA, "verify launch: %s", cudaGetErrorString(e));
  }
  return TL_OK;
}

tl_status tl_storeh_prefill_attn(const tl_storeh_desc* desc, tl_storeh_cache cache, int32_t iter,
                                 const int32_t* loops, const int32_t* ctx_len, const void* h_chunk, int32_t n_tokens,
                                 const void* W_q, const void* W_k, const void* W_v, float* out, void* workspace,
                                 size_t workspace_bytes, int32_t n_lanes, tl_stream_t stream) {
  return tl_storeh_verify_attn(desc, cache, iter, loops, ctx_len, h_chunk, 1, n_tokens, W_q, W_k, W_v, out, workspace,
                               workspace_bytes, n_lanes, stream);
}

}  // extern "C"
