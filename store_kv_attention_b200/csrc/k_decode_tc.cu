// Prologue and epilogue of one store-h decode iteration: the dense projections of the
// absorbed form on tensor cores (k_gemm_tc.cu), with small finishing kernels.
// [Novel Contributions, "Novel Mechanism: Store-h KV Cache": K = W_k h, V = W_v h with
//  the loop block's shared weights]
//
//   prologue : q = W_q h_new                       (GEMM, split-K; q_finish sums the splits)
//              qt_j = W_k[j]^T q_j . log2(e)/sqrt(hd)  (GEMM with A = W_k^T read MN-major,
//              B = q as fp16 hi + lo; qt_finish writes the streaming kernel's operand image)
//   stream   : k_stream_tc.cu, per (lane, split) partials (m, l, U)
//   epilogue : merge the splits exactly: u_j = sum_s 2^(m_s - M) U_s / sum_s 2^(m_s - M) l_s
//              (as fp16 hi + lo), out_j = W_v[j] u_j (GEMM, split-K; o_finish sums the splits)
// Every sum over splits runs in a fixed order, so a lane's result does not depend on the
// other lanes of its batch.
#include <math_constants.h>

#include "tl_internal.cuh"

namespace tl {
namespace {

constexpr int kFinThreads = 256;

__global__ void __launch_bounds__(kFinThreads) q_finish_kernel(Shape s, int iter, const int32_t* __restrict__ loops,
                                                               const int32_t* __restrict__ ctx_len,
                                                               const float* __restrict__ part, int sq, int nb,
                                                               int n_lanes, __half* __restrict__ qhl,
                                                               uint32_t* status) {
  if (blockIdx.x == 0 && threadIdx.x < 32) {
    // range check of the per-lane device values, once per decode call
    for (int b = threadIdx.x; b < n_lanes; b += 32) {
      const int L = loops[b], c = ctx_len[b];
      if (L < 0 || L > s.L_max || c < 0 || c >= s.max_ctx) atomicOr(status, kStatusRange);
    }
  }
  const int idx = blockIdx.x * kFinThreads + threadIdx.x;
  if (idx >= s.d * nb) return;
  const int r = idx / nb, b = idx % nb;
  float q = 0.0f;
  for (int sp = 0; sp < sq; ++sp) q += part[((size_t)sp * s.d + r) * nb + b];
  int n;
  if (b >= n_lanes || !lane_active(s, iter, loops, ctx_len, b, &n)) q = 0.0f;
  const __half hi = __float2half_rn(q);
  qhl[(size_t)b * s.d + r] = hi;
  qhl[(size_t)(nb + b) * s.d + r] = __float2half_rn(q - __half2float(hi));
}

// The B-operand image of the streaming kernel's score MMA: row j = fp16(qt_j), and when the
// operands are split, row 16 + j = fp16(qt_j - fp16(qt_j)); columns in the dequantised position
// order, 128-byte swizzled atom-columns.  Rows of heads j >= H are zero.
__global__ void __launch_bounds__(kFinThreads) qt_finish_kernel(Shape s, int iter, const int32_t* __restrict__ loops,
                                                                const int32_t* __restrict__ ctx_len,
                                                                const float* __restrict__ part, int nb, int n_lanes,
                                                                uint8_t* __restrict__ qimg) {
  const int c = blockIdx.x * kFinThreads + threadIdx.x;
  const int j = blockIdx.y, b = blockIdx.z;
  if (c >= s.d) return;
  int n;
  if (!lane_active(s, iter, loops, ctx_len, b, &n)) return;
  float v = 0.0f;
  if (j < s.H) {
    const float* pr = part + ((size_t)j * s.d + c) * (2 * nb);
    v = (pr[b] + pr[nb + b]) * (1.4426950408889634f / sqrtf((float)s.hd));
  }
  const int rows = qimg_rows(s.d);
  const int pos = phys_pos(s.fmt, c);
  uint8_t* img = qimg + (size_t)b * qimg_bytes(s.d);
  const __half hi = __float2half_rn(v);
  *reinterpret_cast<__half*>(img + kmajor_offset(j, pos, rows)) = hi;
  if (split_operands(s.d))
    *reinterpret_cast<__half*>(img + kmajor_offset(16 + j, pos, rows)) = __float2half_rn(v - __half2float(hi));
}

// Exact merge of a lane's split partials for head j, written as fp16 hi + lo rows of the
// value-projection GEMM's B operand.
__global__ void __launch_bounds__(kFinThreads) merge_kernel(Shape s, int iter, const int32_t* __restrict__ loops,
                                                            const int32_t* __restrict__ ctx_len,
                                                            const float* __restrict__ ml, const float* __restrict__ U,
                                                            int s_max, int nb, __half* __restrict__ uhl) {
  __shared__ float wgt[kMaxSplits];
  const int b = blockIdx.x, j = blockIdx.y;
  int n = 0;
  const bool active = lane_active(s, iter, loops, ctx_len, b, &n);
  const int S = active ? splits_for_rows(n) : 0;
  if (threadIdx.x == 0 && S > 0) {
    float M = -CUDART_INF_F;
    for (int sp = 0; sp < S; ++sp) M = fmaxf(M, ml[(((size_t)b * s_max + sp) * kMaxHeads + j) * 2]);
    float L = 0.0f;
    for (int sp = 0; sp < S; ++sp) {
      const float* p = ml + (((size_t)b * s_max + sp) * kMaxHeads + j) * 2;
      L += p[1] * exp2f(p[0] - M);
    }
    for (int sp = 0; sp < S; ++sp) {
      const float* p = ml + (((size_t)b * s_max + sp) * kMaxHeads + j) * 2;
      wgt[sp] = exp2f(p[0] - M) / L;
    }
  }
  __syncthreads();
  __half* hi_row = uhl + ((size_t)j * 2 * nb + b) * s.d;
  __half* lo_row = uhl + ((size_t)j * 2 * nb + nb + b) * s.d;
  for (int k = threadIdx.x; k < s.d; k += kFinThreads) {
    float v = 0.0f;
    for (int sp = 0; sp < S; ++sp) v = fmaf(wgt[sp], U[(((size_t)b * s_max + sp) * kMaxHeads + j) * s.d + k], v);
    const __half hi = __float2half_rn(v);
    hi_row[k] = hi;
    lo_row[k] = __float2half_rn(v - __half2float(hi));
  }
}

// out[b][j][r] = sum over splits of the hi and lo columns of the value-projection GEMM.
__global__ void __launch_bounds__(kFinThreads) o_finish_kernel(Shape s, int iter, const int32_t* __restrict__ loops,
                                                               const int32_t* __restrict__ ctx_len,
                                                               const float* __restrict__ part, int so, int nb,
                                                               int n_lanes, float* __restrict__ out) {
  const int idx = blockIdx.x * kFinThreads + threadIdx.x;
  if (idx >= n_lanes * s.d) return;
  const int b = idx / s.d, jr = idx % s.d, j = jr / s.hd, r = jr % s.hd;
  int n;
  if (!lane_active(s, iter, loops, ctx_len, b, &n)) return;
  const int ncol = o_cols(s, nb);
  const int z = s.hd == 64 ? j >> 1 : j;
  const int row = s.hd == 64 ? (j & 1) * 64 + r : r;
  const int c0 = s.hd == 64 ? (j & 1) * 2 * nb : 0;
  float v = 0.0f;
  for (int sp = 0; sp < so; ++sp) {
    const float* pr = part + (((size_t)z * so + sp) * 128 + row) * ncol + c0;
    v += pr[b] + pr[nb + b];
  }
  out[(size_t)b * s.d + jr] = v;
}

}  // namespace

cudaError_t launch_prologue(const DecodeArgs& a, cudaStream_t st) {
  const Shape& s = a.s;
  const Workspace& w = a.wl;
  uint32_t* status = reinterpret_cast<uint32_t*>(a.ws + w.status_off);
  float* qpart = reinterpret_cast<float*>(a.ws + w.qpart_off);
  __half* qhl = reinterpret_cast<__half*>(a.ws + w.qhl_off);
  float* qtpart = reinterpret_cast<float*>(a.ws + w.qtpart_off);
  alignas(64) unsigned char tA[128], tB[128];

  // q = W_q h_new: A = W_q [d][d] (K-major), B = h_new [n_lanes][d]; box rows past n_lanes read as zero
  if (!make_tmap_f16(tA, a.Wq, s.d, s.d, s.d, 64, 128) || !make_tmap_f16(tB, a.h_new, a.n_lanes, s.d, s.d, 64, w.nb))
    return cudaErrorInvalidValue;
  cudaError_t e = launch_gemm_tc(false, tA, tB, s.d, w.nb, s.d, w.sq, 1, 0, 0, 0, 0, qpart, status, st);
  if (e != cudaSuccess) return e;
  const int nq = s.d * w.nb;
  q_finish_kernel<<<(nq + kFinThreads - 1) / kFinThreads, kFinThreads, 0, st>>>(s, a.iter, a.loops, a.ctx_len, qpart,
                                                                                w.sq, w.nb, a.n_lanes, qhl, status);
  count_launch();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  // qt_j = W_k[j]^T q_j: A = W_k^T read MN-major (W_k rows j*hd.. are the K range of head j),
  // B = q hi/lo [2 NB][d] (columns j*hd.. of head j); one batch entry per head
  if (!make_tmap_f16(tA, a.Wk, s.d, s.d, s.d, 64, 64) || !make_tmap_f16(tB, qhl, 2 * w.nb, s.d, s.d, 64, 2 * w.nb))
    return cudaErrorInvalidValue;
  e = launch_gemm_tc(true, tA, tB, s.d, 2 * w.nb, s.hd, 1, s.H, 0, s.hd, s.hd, 0, qtpart, status, st);
  if (e != cudaSuccess) return e;
  qt_finish_kernel<<<dim3((s.d + kFinThreads - 1) / kFinThreads, kMaxHeads, a.n_lanes), kFinThreads, 0, st>>>(
      s, a.iter, a.loops, a.ctx_len, qtpart, w.nb, a.n_lanes, a.ws + w.qt_off);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_epilogue(const DecodeArgs& a, cudaStream_t st) {
  const Shape& s = a.s;
  const Workspace& w = a.wl;
  uint32_t* status = reinterpret_cast<uint32_t*>(a.ws + w.status_off);
  __half* uhl = reinterpret_cast<__half*>(a.ws + w.uhl_off);
  float* opart = reinterpret_cast<float*>(a.ws + w.opart_off);
  merge_kernel<<<dim3(a.n_lanes, s.H), kFinThreads, 0, st>>>(s, a.iter, a.loops, a.ctx_len,
                                                             reinterpret_cast<const float*>(a.ws + w.ml_off),
                                                             reinterpret_cast<const float*>(a.ws + w.u_off), w.s_max,
                                                             w.nb, uhl);
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  // out_j = W_v[j] u_j: one 128-row block of W_v per batch entry (one head, or two when hd = 64),
  // B = the matching hi/lo rows of u
  const int ncol = o_cols(s, w.nb);
  alignas(64) unsigned char tA[128], tB[128];
  if (!make_tmap_f16(tA, a.Wv, s.d, s.d, s.d, 64, 128) ||
      !make_tmap_f16(tB, uhl, (uint64_t)s.H * 2 * w.nb, s.d, s.d, 64, ncol))
    return cudaErrorInvalidValue;
  e = launch_gemm_tc(false, tA, tB, 128, ncol, s.d, w.so, s.d / 128, 0, 128, 0, ncol, opart, status, st);
  if (e != cudaSuccess) return e;
  const int no = a.n_lanes * s.d;
  o_finish_kernel<<<(no + kFinThreads - 1) / kFinThreads, kFinThreads, 0, st>>>(s, a.iter, a.loops, a.ctx_len, opart,
                                                                                w.so, w.nb, a.n_lanes, a.out);
  count_launch();
  return cudaGetLastError();
}

}  // namespace tl
