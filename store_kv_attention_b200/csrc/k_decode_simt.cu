// Store-h decode attention, CUDA-core kernels: prologue (query, absorbed query) and epilogue
// (split merge + W_v).  The context-streaming kernel between them is k_stream_tc.cu.
// [Novel Contributions, "Novel Mechanism: Store-h KV Cache"; Architecture-Exclusive
//  Features, "Store-h KV cache", "Variable-L KV cache", "L-aware batching"]
//
// Absorbed form of K = W_k h, V = W_v h for one loop iteration i, layer n_pre+i:
//   prologue : q = W_q h_new ; qt_j = W_k[j]^T q_j * log2(e)/sqrt(hd)   (fp16 operand image, workspace)
//   stream   : (tensor cores, k_stream_tc.cu) per (lane, split): s_cj = qt_j . h_c ;
//              online softmax in base 2 ; U_j = sum_c 2^(s_cj - m_j) h_c  (partials m, l, U)
//   epilogue : merge the splits of a lane exactly ; u_j = U_j / l_j ; out_j = W_v[j] u_j
// The split plan depends only on the lane's own context length, so a lane's
// result does not depend on which other lanes share its batch.
#include <math_constants.h>

#include "tl_internal.cuh"

namespace tl {
namespace {

__device__ __forceinline__ bool lane_active(const Shape& s, int iter, const int32_t* loops, const int32_t* ctx_len,
                                            int b, int* n_rows) {
  const int L = loops[b];
  const int c = ctx_len[b];
  if (L < 0 || L > s.L_max || c < 0 || c >= s.max_ctx) return false;
  if (iter >= L) return false;
  *n_rows = c + 1;
  return true;
}

// ------------------------------------------------------------------ prologue: q
// One warp per output row r of W_q; the warp keeps the row in registers and
// dots it with every lane's h_new.
constexpr int kQWarps = 8;

__global__ void __launch_bounds__(kQWarps * 32) q_kernel(Shape s, int iter, const int32_t* __restrict__ loops,
                                                        const int32_t* __restrict__ ctx_len,
                                                        const __half* __restrict__ h_new,
                                                        const __half* __restrict__ Wq, float* __restrict__ q,
                                                        int n_lanes, uint32_t* status) {
  const int r = blockIdx.x * kQWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (blockIdx.x == 0 && threadIdx.x < 32) {
    // range check of the per-lane device values, once per launch
    for (int b = lane; b < n_lanes; b += 32) {
      const int L = loops[b], c = ctx_len[b];
      if (L < 0 || L > s.L_max || c < 0 || c >= s.max_ctx) atomicOr(status, kStatusRange);
    }
  }
  if (r >= s.d) return;
  const int nv = s.d / 8;  // uint4 (8 halves) per row
  uint4 w[16];
#pragma unroll
  for (int i = 0; i < 16; ++i)
    if (lane + 32 * i < nv) w[i] = reinterpret_cast<const uint4*>(Wq + (size_t)r * s.d)[lane + 32 * i];
  for (int b = 0; b < n_lanes; ++b) {
    int n;
    if (!lane_active(s, iter, loops, ctx_len, b, &n)) continue;
    const uint4* h4 = reinterpret_cast<const uint4*>(h_new + (size_t)b * s.d);
    float acc = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (lane + 32 * i < nv) {
        const uint4 hv = h4[lane + 32 * i];
        const __half2* wp = reinterpret_cast<const __half2*>(&w[i]);
        const __half2* hp = reinterpret_cast<const __half2*>(&hv);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 a = __half22float2(wp[k]), c = __half22float2(hp[k]);
          acc = fmaf(a.x, c.x, acc);
          acc = fmaf(a.y, c.y, acc);
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) q[(size_t)b * s.d + r] = acc;
  }
}

// ------------------------------------------------------------------ prologue: qt
// qt[b][j][c] = sum_{r<hd} W_k[j*hd + r][c] * q[b][j*hd + r], times log2(e)/sqrt(hd), in fp32,
// written as the fp16 B-operand image of the tensor-core scores: row j = fp16(qt), and when the
// operands are split, row 16 + j = fp16(qt - fp16(qt)); columns in the dequantised position order,
// 128-byte swizzled atom-columns.  Heads j >= H are zero rows.
constexpr int kQtThreads = 256;

__global__ void __launch_bounds__(kQtThreads) qt_kernel(Shape s, int iter, const int32_t* __restrict__ loops,
                                                        const int32_t* __restrict__ ctx_len,
                                                        const __half* __restrict__ Wk, const float* __restrict__ q,
                                                        uint8_t* __restrict__ qimg, int n_lanes) {
  const int c = blockIdx.x * kQtThreads + threadIdx.x;
  const int j = blockIdx.y;
  const int rows = qimg_rows(s.d);
  const bool split = split_operands(s.d);
  const int pos = phys_pos(s.fmt, c);
  const float scale = 1.4426950408889634f / sqrtf((float)s.hd);
  for (int b = 0; b < n_lanes; ++b) {
    int n;
    if (!lane_active(s, iter, loops, ctx_len, b, &n)) continue;
    float acc = 0.0f;
    if (j < s.H) {
      const float* qj = q + (size_t)b * s.d + j * s.hd;
      for (int r = 0; r < s.hd; ++r) acc = fmaf(__half2float(Wk[(size_t)(j * s.hd + r) * s.d + c]), qj[r], acc);
      acc *= scale;
    }
    uint8_t* img = qimg + (size_t)b * qimg_bytes(s.d);
    const __half hi = __float2half_rn(acc);
    *reinterpret_cast<__half*>(img + kmajor_offset(j, pos, rows)) = hi;
    if (split) *reinterpret_cast<__half*>(img + kmajor_offset(16 + j, pos, rows)) = __float2half_rn(acc - __half2float(hi));
  }
}

// ------------------------------------------------------------------ epilogue
// Block (head j, group of 8 lanes): merge the lane's splits exactly into
// u = sum_s 2^(m_s - M) U_s / sum_s 2^(m_s - M) l_s, then out_j = W_v[j] u.
constexpr int kEpiLanes = 8;
constexpr int kEpiThreads = 256;

__global__ void __launch_bounds__(kEpiThreads) epilogue_kernel(Shape s, int iter, const int32_t* __restrict__ loops,
                                                               const int32_t* __restrict__ ctx_len,
                                                               const float* __restrict__ ml,
                                                               const float* __restrict__ U,
                                                               const __half* __restrict__ Wv, float* __restrict__ out,
                                                               int n_lanes, int s_max) {
  extern __shared__ float u_sh[];  // [kEpiLanes][d]
  __shared__ float wgt[kEpiLanes][kMaxSplits];
  __shared__ int act[kEpiLanes];
  const int j = blockIdx.x;
  const int b0 = blockIdx.y * kEpiLanes;
  const int d = s.d;
  if (threadIdx.x < kEpiLanes) {
    const int b = b0 + threadIdx.x;
    int n = 0;
    act[threadIdx.x] = (b < n_lanes && lane_active(s, iter, loops, ctx_len, b, &n)) ? splits_for_rows(n) : 0;
    const int S = act[threadIdx.x];
    if (S > 0) {
      float M = -CUDART_INF_F;
      for (int sp = 0; sp < S; ++sp) M = fmaxf(M, ml[(((size_t)b * s_max + sp) * kMaxHeads + j) * 2]);
      float L = 0.0f;
      for (int sp = 0; sp < S; ++sp) {
        const float* p = ml + (((size_t)b * s_max + sp) * kMaxHeads + j) * 2;
        L += p[1] * exp2f(p[0] - M);
      }
      for (int sp = 0; sp < S; ++sp) {
        const float* p = ml + (((size_t)b * s_max + sp) * kMaxHeads + j) * 2;
        wgt[threadIdx.x][sp] = exp2f(p[0] - M) / L;
      }
    }
  }
  __syncthreads();
  for (int lb = 0; lb < kEpiLanes; ++lb) {
    const int S = act[lb];
    if (S == 0) continue;
    const int b = b0 + lb;
    for (int k = threadIdx.x; k < d; k += kEpiThreads) {
      float v = 0.0f;
      for (int sp = 0; sp < S; ++sp) v = fmaf(wgt[lb][sp], U[(((size_t)b * s_max + sp) * kMaxHeads + j) * d + k], v);
      u_sh[lb * d + k] = v;
    }
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int r = warp; r < s.hd; r += kEpiThreads / 32) {
    const __half* wrow = Wv + (size_t)(j * s.hd + r) * d;
    float accs[kEpiLanes];
#pragma unroll
    for (int lb = 0; lb < kEpiLanes; ++lb) accs[lb] = 0.0f;
    for (int k = lane * 2; k < d; k += 64) {
      const float2 w = __half22float2(*reinterpret_cast<const __half2*>(wrow + k));
#pragma unroll
      for (int lb = 0; lb < kEpiLanes; ++lb) {
        accs[lb] = fmaf(w.x, u_sh[lb * d + k], accs[lb]);
        accs[lb] = fmaf(w.y, u_sh[lb * d + k + 1], accs[lb]);
      }
    }
#pragma unroll
    for (int lb = 0; lb < kEpiLanes; ++lb) {
      float v = accs[lb];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0 && act[lb] > 0) out[((size_t)(b0 + lb) * s.H + j) * s.hd + r] = v;
    }
  }
}

}  // namespace

cudaError_t launch_prologue(const DecodeArgs& a, cudaStream_t st) {
  const Shape& s = a.s;
  float* q = reinterpret_cast<float*>(a.ws + a.wl.q_off);
  uint8_t* qt = a.ws + a.wl.qt_off;
  uint32_t* status = reinterpret_cast<uint32_t*>(a.ws + a.wl.status_off);
  q_kernel<<<(s.d + kQWarps - 1) / kQWarps, kQWarps * 32, 0, st>>>(s, a.iter, a.loops, a.ctx_len, a.h_new, a.Wq, q,
                                                                  a.n_lanes, status);
  count_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  qt_kernel<<<dim3(s.d / kQtThreads, kMaxHeads), kQtThreads, 0, st>>>(s, a.iter, a.loops, a.ctx_len, a.Wk, q, qt,
                                                                        a.n_lanes);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_epilogue(const DecodeArgs& a, cudaStream_t st) {
  const Shape& s = a.s;
  const size_t sm = (size_t)kEpiLanes * s.d * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(epilogue_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  dim3 grid(s.H, (a.n_lanes + kEpiLanes - 1) / kEpiLanes);
  epilogue_kernel<<<grid, kEpiThreads, sm, st>>>(s, a.iter, a.loops, a.ctx_len,
                                                 reinterpret_cast<const float*>(a.ws + a.wl.ml_off),
                                                 reinterpret_cast<const float*>(a.ws + a.wl.u_off), a.Wv, a.out,
                                                 a.n_lanes, a.wl.s_max);
  count_launch();
  return cudaGetLastError();
}

}  // namespace tl
