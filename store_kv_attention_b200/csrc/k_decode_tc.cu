// Prologue and epilogue of one store-h decode iteration: the dense projections of the
// absorbed form on tensor cores (k_gemm_tc.cu), with small finishing kernels.
// [Novel Contributions, "Novel Mechanism: Store-h KV Cache": K = W_k h, V = W_v h with
//  the loop block's shared weights]
//
//   prologue : q = W_q h_new                       (GEMM, split-K; its last CTA per block sums the splits)
//              qt_j = W_k[j]^T q_j . log2(e)/sqrt(hd)  (GEMM with A = W_k^T read MN-major,
//              B = q as fp16 hi + lo; its epilogue writes the streaming kernel's operand image)
//   stream   : k_stream_tc.cu, per (lane, split) partials (m, l, U)
//   epilogue : merge the splits exactly: u_j = sum_s 2^(m_s - M) U_s / sum_s 2^(m_s - M) l_s
//              (as fp16 hi + lo), out_j = W_v[j] u_j (GEMM, split-K; its last CTA per block sums the splits)
// Every sum over splits runs in a fixed order, so a lane's result does not depend on the
// other lanes of its batch.
#include <math_constants.h>

#include "norm_block.cuh"
#include "tl_internal.cuh"

namespace tl {
namespace {

constexpr int kFinThreads = 256;

// Exact merge of a lane's split partials for head j, written as fp16 hi + lo rows of the
// value-projection GEMM's B operand:  u_j = sum_s 2^(m_s - M) U_s / sum_s 2^(m_s - M) l_s.
// Blocks with blockIdx.y == H run the per-iteration safety check of lane blockIdx.x instead
// (it depends only on the residual, so it shares this launch).
struct MergeArgs {
  Shape s;
  int iter;
  const int32_t* loops;
  const int32_t* ctx_len;
  const float* ml;
  const float* U;
  int s_max, nb;
  __half* uhl;
  const float* residual;
  float threshold;
  uint8_t* flags;
  int32_t* first;
  float* norms;
};

__global__ void __launch_bounds__(kFinThreads) merge_kernel(const MergeArgs g) {
  __shared__ float wgt[kMaxSplits];
  const Shape& s = g.s;
  const int b = blockIdx.x, j = blockIdx.y;
  int n = 0;
  const bool active = lane_active(s, g.iter, g.loops, g.ctx_len, b, &n);
  if (j == s.H) {
    if (active) norm_check_lane<kFinThreads>(g.residual, b, s.d, g.threshold, g.iter, g.flags, g.first, g.norms);
    return;
  }
  const int S = active ? splits_for_rows(n) : 0;
  if (threadIdx.x == 0 && S > 0) {
    float M = -CUDART_INF_F;
    for (int sp = 0; sp < S; ++sp) M = fmaxf(M, g.ml[(((size_t)b * g.s_max + sp) * kMaxHeads + j) * 2]);
    float L = 0.0f;
    for (int sp = 0; sp < S; ++sp) {
      const float* p = g.ml + (((size_t)b * g.s_max + sp) * kMaxHeads + j) * 2;
      L += p[1] * exp2f(p[0] - M);
    }
    for (int sp = 0; sp < S; ++sp) {
      const float* p = g.ml + (((size_t)b * g.s_max + sp) * kMaxHeads + j) * 2;
      wgt[sp] = exp2f(p[0] - M) / L;
    }
  }
  __syncthreads();
  __half* hi_row = g.uhl + ((size_t)j * 2 * g.nb + b) * s.d;
  __half* lo_row = g.uhl + ((size_t)j * 2 * g.nb + g.nb + b) * s.d;
  const float* U0 = g.U + ((size_t)b * g.s_max * kMaxHeads + j) * s.d;  // split sp at + sp * 16 * d
  for (int k4 = threadIdx.x; k4 < s.d / 4; k4 += kFinThreads) {
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int sp0 = 0; sp0 < S; sp0 += 8) {
      float4 t[8];
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (sp0 + k < S) t[k] = __ldcs(reinterpret_cast<const float4*>(U0 + (size_t)(sp0 + k) * kMaxHeads * s.d) + k4);
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (sp0 + k < S) {
          const float w = wgt[sp0 + k];
          v.x = fmaf(w, t[k].x, v.x);
          v.y = fmaf(w, t[k].y, v.y);
          v.z = fmaf(w, t[k].z, v.z);
          v.w = fmaf(w, t[k].w, v.w);
        }
    }
    const float vv[4] = {v.x, v.y, v.z, v.w};
    __align__(8) __half h[4], l[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      h[i] = __float2half_rn(vv[i]);
      l[i] = __float2half_rn(vv[i] - __half2float(h[i]));
    }
    *reinterpret_cast<uint2*>(hi_row + 4 * k4) = *reinterpret_cast<const uint2*>(h);
    *reinterpret_cast<uint2*>(lo_row + 4 * k4) = *reinterpret_cast<const uint2*>(l);
  }
}

}  // namespace

GemmEpiParams epi_params(const DecodeArgs& a, int mode) {
  GemmEpiParams e{};
  e.mode = mode;
  e.s = a.s;
  e.iter = a.iter;
  e.loops = a.loops;
  e.ctx_len = a.ctx_len;
  e.n_lanes = a.n_lanes;
  e.nb = a.wl.nb;
  e.status = reinterpret_cast<uint32_t*>(a.ws + a.wl.status_off);
  e.counters = reinterpret_cast<uint32_t*>(a.ws + a.wl.status_off + (mode == kEpiOut ? kCountersOOff : kCountersQOff));
  e.qhl = reinterpret_cast<__half*>(a.ws + a.wl.qhl_off);
  e.qimg = a.ws + a.wl.qt_off;
  e.out = a.out;
  return e;
}

cudaError_t launch_prologue(const DecodeArgs& a, cudaStream_t st) {
  const Shape& s = a.s;
  const Workspace& w = a.wl;
  uint32_t* status = reinterpret_cast<uint32_t*>(a.ws + w.status_off);
  float* qpart = reinterpret_cast<float*>(a.ws + w.qpart_off);
  __half* qhl = reinterpret_cast<__half*>(a.ws + w.qhl_off);
  float* qtpart = reinterpret_cast<float*>(a.ws + w.qtpart_off);
  alignas(64) unsigned char tA[128], tB[128];

  // q = W_q h_new: A = W_q [d][d] (K-major), B = h_new [n_lanes][d]; box rows past n_lanes read as zero.
  // The last CTA of each row block sums the K splits and writes q as fp16 hi/lo rows.
  if (!make_tmap_f16(tA, a.Wq, s.d, s.d, s.d, 64, 128) || !make_tmap_f16(tB, a.h_new, a.n_lanes, s.d, s.d, 64, w.nb))
    return cudaErrorInvalidValue;
  cudaError_t e = launch_gemm_tc(false, tA, tB, s.d, w.nb, s.d, w.sq, 1, 0, 0, 0, 0, qpart, status,
                                 epi_params(a, kEpiQ), st);
  if (e != cudaSuccess) return e;

  // qt_j = W_k[j]^T q_j: A = W_k^T read MN-major (W_k rows j*hd.. are the K range of head j),
  // B = q hi/lo [2 NB][d] (columns j*hd.. of head j); one batch entry per head.  The epilogue
  // writes the streaming kernel's operand image.
  if (!make_tmap_f16(tA, a.Wk, s.d, s.d, s.d, 64, 64) || !make_tmap_f16(tB, qhl, 2 * w.nb, s.d, s.d, 64, 2 * w.nb))
    return cudaErrorInvalidValue;
  return launch_gemm_tc(true, tA, tB, s.d, 2 * w.nb, s.hd, 1, s.H, 0, s.hd, s.hd, 0, qtpart, status,
                        epi_params(a, kEpiQImage), st);
}

cudaError_t launch_epilogue(const DecodeArgs& a, cudaStream_t st) {
  const Shape& s = a.s;
  const Workspace& w = a.wl;
  uint32_t* status = reinterpret_cast<uint32_t*>(a.ws + w.status_off);
  __half* uhl = reinterpret_cast<__half*>(a.ws + w.uhl_off);
  float* opart = reinterpret_cast<float*>(a.ws + w.opart_off);
  const MergeArgs g{s,        a.iter,     a.loops,
                    a.ctx_len,
                    reinterpret_cast<const float*>(a.ws + w.ml_off),
                    reinterpret_cast<const float*>(a.ws + w.u_off),
                    w.s_max,  w.nb,       uhl,
                    a.residual,
                    a.threshold,
                    a.abort_flags,
                    a.first_abort_iter,
                    a.norms};
  merge_kernel<<<dim3(a.n_lanes, s.H + (a.residual ? 1 : 0)), kFinThreads, 0, st>>>(g);
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  // out_j = W_v[j] u_j: one 128-row block of W_v per batch entry (one head, or two when hd = 64),
  // B = the matching hi/lo rows of u; the last CTA of each block sums the K splits into out.
  const int ncol = o_cols(s, w.nb);
  alignas(64) unsigned char tA[128], tB[128];
  if (!make_tmap_f16(tA, a.Wv, s.d, s.d, s.d, 64, 128) ||
      !make_tmap_f16(tB, uhl, (uint64_t)s.H * 2 * w.nb, s.d, s.d, 64, ncol))
    return cudaErrorInvalidValue;
  return launch_gemm_tc(false, tA, tB, 128, ncol, s.d, w.so, s.d / 128, 0, 128, 0, ncol, opart, status,
                        epi_params(a, kEpiOut), st);
}

}  // namespace tl
