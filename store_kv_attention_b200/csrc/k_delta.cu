// Iteration-axis delta cache of h: the writer.
// [Architecture-Exclusive Features, "Iteration-axis delta-KV": an fp16 anchor per token and,
//  per loop iteration, an INT8 dh with an fp16 per-head scale; h^i rebuilt by an FP32 prefix
//  sum]
//
// One CTA of 128 threads per (row, lane); thread t owns the 16 consecutive elements
// [16 t, 16 t + 16) of the row, so the hd / 16 threads of one head (4 or 8 lanes, aligned
// within a warp) reduce its amax by shuffles.  Iteration 0 stores the row as the anchor.
// Iteration i >= 1 rebuilds h^(i-1) of the position in FP32 (anchor, then deltas 1..i-1 in
// order, one rounding per addition; each scale * code product is exact), forms
// dh = h^i - rebuild, and quantises it per head:
//   scale = fp16_rne(amax / 127.0f), code = clamp(rne(dh / float(scale)), -127, 127),
// with IEEE divisions, so the codes and scales are bit-exact to the definition.
#include "delta_internal.cuh"
#include "tc_ptx.cuh"
#include "tl_internal.cuh"

namespace tl {
namespace {

constexpr int kDThreads = 128;  // 16 elements per thread: d <= 2048

__device__ __forceinline__ void load16_f32(const __half* p, float* v) {
  const uint4 a = *reinterpret_cast<const uint4*>(p);
  const uint4 c = *reinterpret_cast<const uint4*>(p + 8);
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

__global__ void __launch_bounds__(kDThreads)
    delta_append_kernel(DeltaShape s, __half* anchor, int8_t* deltas, __half* scales, int iter,
                        const __half* __restrict__ h_rows, int n_rows, const int32_t* __restrict__ start_pos,
                        const int32_t* __restrict__ loops) {
  ptx::pdl_wait();  // the rows may come from the previous kernel in the stream
  ptx::pdl_trigger();
  const int r = blockIdx.x, b = blockIdx.y;
  if (loops && iter >= loops[b]) return;  // the same for the whole CTA
  const long long pos = (long long)start_pos[b] + r;
  if (pos < 0 || pos >= s.max_ctx) return;
  const int k0 = threadIdx.x * 16;
  const bool active = k0 < s.d;  // d is a multiple of 256: whole heads are active or not
  const size_t row = (size_t)b * s.max_ctx + (size_t)pos;
  const size_t level_rows = (size_t)s.max_lanes * s.max_ctx;
  const __half* src = h_rows + ((size_t)b * n_rows + r) * s.d;

  if (iter == 0) {
    if (active) {
      const uint4* in = reinterpret_cast<const uint4*>(src + k0);
      uint4* out = reinterpret_cast<uint4*>(anchor + row * s.d + k0);
      out[0] = in[0];
      out[1] = in[1];
    }
    return;
  }

  float h[16], acc[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) h[j] = acc[j] = 0.0f;
  const int head = active ? k0 / s.hd : 0;
  if (active) {
    load16_f32(src + k0, h);
    load16_f32(anchor + row * s.d + k0, acc);
    for (int i = 1; i < iter; ++i) {
      const size_t lr = (size_t)(i - 1) * level_rows + row;
      const uint4 cv = *reinterpret_cast<const uint4*>(deltas + lr * s.d + k0);
      const float sc = __half2float(scales[lr * s.H + head]);
      const int8_t* c = reinterpret_cast<const int8_t*>(&cv);
#pragma unroll
      for (int j = 0; j < 16; ++j) acc[j] = __fadd_rn(acc[j], __fmul_rn((float)c[j], sc));
    }
  }
  float dh[16], amax = 0.0f;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    dh[j] = __fsub_rn(h[j], acc[j]);
    amax = fmaxf(amax, fabsf(dh[j]));
  }
  for (int o = 1; o < s.hd / 16; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const __half s16 = __float2half_rn(__fdiv_rn(amax, 127.0f));
  const float div = __half2float(s16);
  uint32_t packed[4];
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    uint32_t v = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int q = 0;
      if (div > 0.0f) q = min(127, max(-127, __float2int_rn(__fdiv_rn(dh[4 * w + j], div))));
      v |= (uint32_t)(q & 0xFF) << (8 * j);
    }
    packed[w] = v;
  }
  if (active) {
    const size_t lw = (size_t)(iter - 1) * level_rows + row;
    *reinterpret_cast<uint4*>(deltas + lw * s.d + k0) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    if ((threadIdx.x & (s.hd / 16 - 1)) == 0) scales[lw * s.H + head] = s16;
  }
}

// Per-lane values of one delta decode call: a lane whose loops / ctx_len are out of range is
// recorded in the status word and skipped; wloops = the writer's loop count (0 = write
// nothing), dloops = the decode's (1 when the lane attends at this iteration, else 0).
__global__ void delta_prep_kernel(int iter, int L_max, int max_ctx, int n_lanes, const int32_t* __restrict__ loops,
                                  const int32_t* __restrict__ ctx_len, int32_t* wloops, int32_t* dloops,
                                  uint32_t* status) {
  ptx::pdl_wait();
  ptx::pdl_trigger();
  const int b = threadIdx.x;
  if (b >= n_lanes) return;
  const int L = loops[b], c = ctx_len[b];
  const bool ok = L >= 0 && L <= L_max && c >= 0 && c < max_ctx;
  if (!ok) atomicOr(status, kStatusRange);
  wloops[b] = ok ? L : 0;
  dloops[b] = ok && iter < L ? 1 : 0;
}

}  // namespace

cudaError_t launch_delta_prep(int iter, int L_max, int max_ctx, int n_lanes, const int32_t* loops,
                              const int32_t* ctx_len, int32_t* wloops, int32_t* dloops, uint32_t* status,
                              cudaStream_t st) {
  if (n_lanes > 1024) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1, 1, 1);
  cfg.blockDim = dim3(((n_lanes + 31) / 32) * 32, 1, 1);
  cfg.stream = st;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, delta_prep_kernel, iter, L_max, max_ctx, n_lanes, loops, ctx_len, wloops,
                                     dloops, status);
  count_launch();
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_delta_append(const DeltaShape& s, void* anchor, void* deltas, void* scales, int iter,
                                const __half* h_rows, int n_lanes, int n_rows, const int32_t* start_pos,
                                const int32_t* loops, cudaStream_t st) {
  if (n_lanes > 65535) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_rows, n_lanes, 1);
  cfg.blockDim = dim3(kDThreads, 1, 1);
  cfg.stream = st;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, delta_append_kernel, s, (__half*)anchor, (int8_t*)deltas, (__half*)scales,
                                     iter, h_rows, n_rows, start_pos, loops);
  count_launch();
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace tl
