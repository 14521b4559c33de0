// RoPE-compatible variant of store-h decode attention: the scores with rotary position
// embeddings, on 5th-generation tensor cores (tcgen05 + TMEM), sm_100a.
// [Novel Contributions, "Novel Mechanism: Store-h KV Cache": K = W_k h rebuilt from the cached
//  h; the pages give no positional encoding, and this variant applies the standard rotary one]
//
// A rotary embedding rotates q and every K row by angles that depend on their positions, between
// the rebuild K = W_k h and the score, so the absorbed query of the store-h decode no longer
// applies to K: every attended row needs its K rebuilt explicitly, a dense [rows x d] x [d x d]
// contraction.  Three kernels:
//   rope_table_kernel   cos / sin of position * base^(-2i/hd) for i < hd/2, evaluated in FP64
//                       (full range reduction) and stored as fp32 pairs
//   rope_query_kernel   q = W_q h_new per lane (fp32), rotated to the query's position and scaled
//                       by log2(e)/sqrt(hd) (the softmax runs in base 2)
//   rope_score_kernel   per (lane, 128-row tile, block of up to 512 K columns): K = h W_k^T with
//                       tcgen05 (A = the tile's rows dequantised into shared memory, B = W_k
//                       tiles by TMA, D in TMEM), then in the epilogue every row rotates its K by
//                       its own position and takes the dot product with each head's rotated q
// The value side is not rotated, so the streaming kernel's P.V stage and the split merge run as
// in the decode, with these scores given (k_stream_tc.cu, k_proj_tc.cu).
//
// Rotary form ("rotate half" pairing): for head vector x at position t and i < hd/2,
//   x'_i = x_i cos(t theta_i) - x_{i+hd/2} sin(t theta_i),
//   x'_{i+hd/2} = x_{i+hd/2} cos(t theta_i) + x_i sin(t theta_i),   theta_i = base^(-2i/hd).
// Row c sits at position c; the query of a lane with ctx_len cached positions at position ctx_len.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "tc_ptx.cuh"
#include "tl_internal.cuh"

namespace tl {
namespace {

using namespace ptx;

constexpr int kRThreads = 256;  // two threads per row of the tile, one per half of each 64-value K slice
constexpr int kATile = 128 * 64 * 2;  // 128 rows x 64 fp16, K-major, 128-byte swizzle
constexpr long long kRWait = 4000000000ll;

__global__ void rope_table_kernel(int rows, int half, int hd, double base, float2* cs) {
  ptx::pdl_wait();
  ptx::pdl_trigger();
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= rows * half) return;
  // angle index major: [half][rows], so the rows of a tile read consecutive entries
  const int i = idx / rows, c = idx % rows;
  const double theta = pow(base, -2.0 * (double)i / (double)hd);
  double sn, cn;
  sincos((double)c * theta, &sn, &cn);
  cs[idx] = make_float2((float)cn, (float)sn);
}

// grid (n_heads, n_lanes), block 128: warp w computes rows w, w + 4, ... of the head with the
// lanes striding over d, then the head is rotated to the lane's query position.
__global__ void rope_query_kernel(Shape s, int iter, const int32_t* loops, const int32_t* ctx_len,
                                  const __half* __restrict__ h_new, const __half* __restrict__ Wq, const float2* cs,
                                  float* qrot) {
  ptx::pdl_wait();
  ptx::pdl_trigger();
  const int j = blockIdx.x, b = blockIdx.y;
  int nr;
  if (!lane_active(s, iter, loops, ctx_len, b, &nr)) return;
  __shared__ float q[128];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const __half* h = h_new + (size_t)b * s.d;
  for (int m = warp; m < s.hd; m += 4) {
    const __half* w = Wq + (size_t)(j * s.hd + m) * s.d;
    float acc = 0.0f;
    for (int k = lane * 8; k < s.d; k += 256) {
      const uint4 wv = *reinterpret_cast<const uint4*>(w + k);
      const uint4 hv = *reinterpret_cast<const uint4*>(h + k);
      const __half2* w2 = reinterpret_cast<const __half2*>(&wv);
      const __half2* h2 = reinterpret_cast<const __half2*>(&hv);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 a = __half22float2(w2[i]), c = __half22float2(h2[i]);
        acc = fmaf(a.x, c.x, acc);
        acc = fmaf(a.y, c.y, acc);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) q[m] = acc;
  }
  __syncthreads();
  const int half = s.hd / 2;
  const float scale = 1.4426950408889634f / sqrtf((float)s.hd);
  const int pos = ctx_len[b];  // the query's position (its own row)
  for (int i = threadIdx.x; i < half; i += blockDim.x) {
    const float2 c = cs[(size_t)i * s.max_ctx + pos];
    const float x1 = q[i], x2 = q[i + half];
    qrot[(size_t)b * s.d + j * s.hd + i] = (x1 * c.x - x2 * c.y) * scale;
    qrot[(size_t)b * s.d + j * s.hd + i + half] = (x2 * c.x + x1 * c.y) * scale;
  }
}

struct RopeScoreParams {
  Shape s;
  int iter;
  const int32_t* loops;
  const int32_t* ctx_len;
  const uint8_t* codes;
  const uint8_t* scales;
  const float* qrot;   // [n_lanes][d]
  const float2* cs;    // [max_ctx][hd/2]
  float* scores;       // [n_lanes][max_ctx][16]
  uint32_t* status;
  int n_pass;          // K columns per CTA (a multiple of hd, at most 512)
};

// The raw codes of the 32 values [k0, k0 + 32) of one cached row (and, for INT4, their group
// scale), loaded one K-step ahead of their use so that the loads are in flight during the MMAs.
struct RowSlice {
  uint4 v[4];
  __half sc;
};
__device__ __forceinline__ void load_row(const Shape& s, const uint8_t* codes, const uint8_t* scales, size_t row,
                                         bool valid, int k0, RowSlice& x) {
  if (!valid) return;
  if (s.fmt == TL_H_FP16) {
    const uint4* src = reinterpret_cast<const uint4*>(codes + row * (size_t)(2 * s.d) + 2 * k0);
#pragma unroll
    for (int v = 0; v < 4; ++v) x.v[v] = __ldg(src + v);
  } else if (s.fmt == TL_H_INT8_TOKEN) {
    const uint4* src = reinterpret_cast<const uint4*>(codes + row * (size_t)s.d + k0);
    x.v[0] = __ldg(src);
    x.v[1] = __ldg(src + 1);
  } else {
    x.v[0] = __ldg(reinterpret_cast<const uint4*>(codes + row * (size_t)(s.d / 2) + k0 / 2));
    x.sc = reinterpret_cast<const __half*>(scales)[row * (size_t)(s.d / kInt4Group) + k0 / kInt4Group];
  }
}

// The loaded slice as fp16 pairs into half `hf` of row r of a K-major swizzled A tile, in the
// natural K order.  FP16 rows are copied; INT8 codes and INT4 codes are converted exactly by the
// exponent-bias ("magic number") identity of IEEE binary16 (a small integer n in the low
// mantissa bits of 2^10 reads as 1024 + n; the method as used for INT4/INT8 dequantisation is
// described by Kim et al., "Who Says Elephants Can't Run", arXiv:2211.10017), INT4 then
// multiplied by its group scale (rounded once to fp16); the INT8 row scale is applied to the
// scores.  Rows outside the lane give zeros.
__device__ __forceinline__ void stage_row(const Shape& s, const RowSlice& x, bool valid, uint8_t* tile, int r, int hf) {
  uint32_t h[16];
  if (!valid) {
#pragma unroll
    for (int i = 0; i < 16; ++i) h[i] = 0u;
  } else if (s.fmt == TL_H_FP16) {
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      h[4 * v] = x.v[v].x;
      h[4 * v + 1] = x.v[v].y;
      h[4 * v + 2] = x.v[v].z;
      h[4 * v + 3] = x.v[v].w;
    }
  } else if (s.fmt == TL_H_INT8_TOKEN) {
    const __half2 bias = __halves2half2(__float2half_rn(1152.0f), __float2half_rn(1152.0f));
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      const uint32_t w[4] = {x.v[v].x, x.v[v].y, x.v[v].z, x.v[v].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t y = w[q] ^ 0x80808080u;            // offset binary: code + 128
        const uint32_t a = prmt(y, 0x64646464u, 0x5140u);  // (1024 + b0, 1024 + b1)
        const uint32_t c = prmt(y, 0x64646464u, 0x7362u);  // (b2, b3)
        const __half2 ha = __hsub2(*reinterpret_cast<const __half2*>(&a), bias);
        const __half2 hc = __hsub2(*reinterpret_cast<const __half2*>(&c), bias);
        h[8 * v + 2 * q] = *reinterpret_cast<const uint32_t*>(&ha);
        h[8 * v + 2 * q + 1] = *reinterpret_cast<const uint32_t*>(&hc);
      }
    }
  } else {
    const __half2 s2 = __halves2half2(x.sc, x.sc);
    const __half2 bias = __halves2half2(__float2half_rn(1032.0f), __float2half_rn(1032.0f));
    const uint32_t w[4] = {x.v[0].x, x.v[0].y, x.v[0].z, x.v[0].w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {  // word q: values 8 q .. 8 q + 7, low nibble first
      const uint32_t t = w[q] & 0x0F0F0F0Fu, u = (w[q] >> 4) & 0x0F0F0F0Fu;  // even / odd values
      const uint32_t sel[4] = {0x4400u, 0x5511u, 0x6622u, 0x7733u};           // pair (2k, 2k + 1)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        // (nibble ^ 8) = code + 8 in the mantissa of 1024: 1032 + code, exact
        const uint32_t pr = lop3_and_xor(prmt(t, u, sel[k]), 0x000F000Fu, 0x64086408u);
        const __half2 y = __hmul2(__hsub2(*reinterpret_cast<const __half2*>(&pr), bias), s2);
        h[4 * q + k] = *reinterpret_cast<const uint32_t*>(&y);
      }
    }
  }
#pragma unroll
  for (int v = 0; v < 4; ++v)
    *reinterpret_cast<uint4*>(tile + r * 128 + (((4 * hf + v) ^ (r & 7)) << 4)) =
        make_uint4(h[4 * v], h[4 * v + 1], h[4 * v + 2], h[4 * v + 3]);
}

__device__ __forceinline__ bool block_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  const bool w = mbar_wait(bar, parity, abort, kRWait);
  return __syncthreads_and(w) != 0;
}

// grid (tiles of 128 rows, column blocks of n_pass, lanes), block 256: thread t takes row
// r = t & 127 of the tile and half t >> 7 of each 64-value K slice
__global__ void __launch_bounds__(kRThreads, 1)
    rope_score_kernel(const __grid_constant__ CUtensorMap tmWk, const RopeScoreParams p) {
  const Shape& s = p.s;
  pdl_wait();
  const int tile = blockIdx.x, cb = blockIdx.y, b = blockIdx.z;
  int n;
  if (!lane_active(s, p.iter, p.loops, p.ctx_len, b, &n)) return;
  if (tile * 128 >= n) return;
  const int NP = p.n_pass;
  const int n_ks = s.d / 64;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
  uint8_t* A[2] = {base, base + kATile};
  uint8_t* B[2] = {base + 2 * kATile, base + 2 * kATile + NP * 128};
  float* qs = reinterpret_cast<float*>(base + 2 * kATile + 2 * NP * 128);  // this block's NP rotated q values
  __shared__ uint64_t full[2], empty[2], fin;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, r = threadIdx.x & 127, hf = threadIdx.x >> 7;
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;  // TMEM lane quarter of the warp = rows r
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(&fin, 1);
    abort_flag = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmWk);
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base, NP <= 256 ? 256 : 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_base;
  volatile int* abort_p = &abort_flag;
  pdl_trigger();  // TMEM is held

  for (int i = threadIdx.x; i < NP; i += kRThreads) qs[i] = p.qrot[(size_t)b * s.d + cb * NP + i];
  const int row = tile * 128 + r;
  const bool valid = row < n;
  const size_t grow = ((size_t)(s.n_pre + p.iter) * s.max_lanes + b) * s.max_ctx + (size_t)row;
  const uint32_t idesc = idesc_f16_f32(128, 256, false, false);
  bool ok = true, issued = false;
  // W_k tiles of K-step k go into stage k & 1.  Step k stages its A slice while the MMAs of step
  // k - 1 run, issues its own MMAs, then waits for those of step k - 1 and loads the W_k tiles of
  // step k + 1 into the stage they freed, so each W_k load has a whole MMA period to land.
  int b_issued = 0;  // W_k loads issued (K-steps 0 .. b_issued - 1)
  auto load_b = [&](int ks) {
    const int st = ks & 1;
    mbar_expect_tx(&full[st], (uint32_t)NP * 128);
    for (int nb = 0; nb < NP / 128; ++nb) tma_load_2d(B[st] + nb * 16384, &tmWk, ks * 64, cb * NP + nb * 128, &full[st]);
  };
  if (threadIdx.x == 0) {
    load_b(0);
    b_issued = 1;
  }
  RowSlice nxt;
  load_row(s, p.codes, p.scales, grow, valid, 32 * hf, nxt);
  for (int ks = 0; ks < n_ks && ok; ++ks) {
    const int st = ks & 1, use = ks >> 1;
    // A[st] was last read by the MMAs of step ks - 2, waited for at step ks - 1
    stage_row(s, nxt, valid, A[st], r, hf);
    if (ks + 1 < n_ks) load_row(s, p.codes, p.scales, grow, valid, (ks + 1) * 64 + 32 * hf, nxt);  // in flight during the MMAs
    fence_proxy_async_smem();
    __syncthreads();
    if (warp == 0) {
      const bool got = __all_sync(0xffffffffu, mbar_wait(&full[st], use & 1, abort_p, kRWait));
      if (got) {
        tc_fence_after();
        if (elect_one()) {
          const uint64_t ad = sdesc_sw128(smem_addr(A[st]), 16, 1024);
          for (int nh = 0; nh < NP / 256 + (NP % 256 ? 1 : 0); ++nh) {
            const uint64_t bd = sdesc_sw128(smem_addr(B[st] + nh * 256 * 128), 16, 1024);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss(tbase + nh * 256, ad + (uint64_t)((kk * 32) >> 4), bd + (uint64_t)((kk * 32) >> 4), idesc,
                     (ks | kk) != 0);
          }
          mma_commit(&empty[st]);
        }
        __syncwarp();
      }
    }
    issued = true;
    if (!(ok = __syncthreads_and(!*abort_p) != 0)) break;
    // the MMAs of step ks - 1 are done: stage st ^ 1 is free for the W_k tiles of step ks + 1
    if (ks >= 1 && !(ok = block_wait(&empty[st ^ 1], ((ks - 1) >> 1) & 1, abort_p))) break;
    if (threadIdx.x == 0 && ks + 1 < n_ks) {
      load_b(ks + 1);
      b_issued = ks + 2;
    }
  }
  // the last K-step's MMAs complete on empty[(n_ks - 1) & 1]
  if (ok) ok = block_wait(&empty[(n_ks - 1) & 1], ((n_ks - 1) >> 1) & 1, abort_p);

  if (ok) {
    // every thread of a warp runs the TMEM loads (they are warp-collective); rows past the
    // lane's end read position 0's angles and store nothing
    tc_fence_after();
    const int half = s.hd / 2;
    const float2* cs = p.cs + (valid ? row : 0);  // entry i of this row at cs[i * max_ctx]
    const float sr = (s.fmt == TL_H_INT8_TOKEN && valid) ? reinterpret_cast<const float*>(p.scales)[grow] : 1.0f;
    for (int h = hf; h < NP / s.hd; h += 2) {  // the two warps of a lane quarter take alternate heads
      float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // four chains, summed in a fixed order
      for (int i0 = 0; i0 < half; i0 += 16) {
        uint32_t k1[16], k2[16];
        tmem_ld16(tbase + lane_off + h * s.hd + i0, k1);
        tmem_ld16(tbase + lane_off + h * s.hd + half + i0, k2);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 c = cs[(size_t)(i0 + i) * s.max_ctx];
          const float a1 = __uint_as_float(k1[i]), a2 = __uint_as_float(k2[i]);
          const float r1 = a1 * c.x - a2 * c.y, r2 = a2 * c.x + a1 * c.y;
          acc[i & 3] = fmaf(qs[h * s.hd + i0 + i], r1, acc[i & 3]);
          acc[i & 3] = fmaf(qs[h * s.hd + half + i0 + i], r2, acc[i & 3]);
        }
      }
      const int j = (cb * NP) / s.hd + h;
      if (valid) p.scores[((size_t)b * s.max_ctx + row) * kMaxHeads + j] = ((acc[0] + acc[1]) + (acc[2] + acc[3])) * sr;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && abort_flag) atomicOr(p.status, kStatusTimeout);
  if (warp == 0) {
    if (issued && !ok) {
      // an abandoned pipeline: nothing may still be writing TMEM when it is freed
      if (elect_one()) mma_commit(&fin);  // arrives once every MMA this warp issued is done
      __syncwarp();
      const long long t0 = clock64();
      while (!mbar_try_wait(&fin, 0) && clock64() - t0 < kRWait) {
      }
    }
    if (!ok && threadIdx.x == 0)
      // nor may a W_k load still be writing shared memory when the CTA exits: the latest load of
      // each stage (bounded waits)
      for (int k = b_issued - 1; k >= 0 && k >= b_issued - 2; --k) {
        const long long t1 = clock64();
        while (!mbar_try_wait(&full[k & 1], (k >> 1) & 1) && clock64() - t1 < kRWait) {
        }
      }
    tc_fence_after();
    tmem_dealloc(tbase, NP <= 256 ? 256 : 512);
  }
}

}  // namespace

bool make_tmap_f16(void* tmap, const void* base, uint64_t rows, uint64_t cols, uint64_t pitch_elems,
                   uint32_t box_cols, uint32_t box_rows);

// Output columns of K per CTA: 512 where they divide d_model, else 256 (d_model is a multiple of 256).
int rope_pass_cols(const Shape& s) { return s.d % 512 == 0 ? 512 : 256; }

cudaError_t launch_rope_scores(const DecodeArgs& a, float rope_base, float2* cs, float* qrot, float* scores,
                               cudaStream_t st) {
  const Shape& s = a.s;
  const int half = s.hd / 2;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.stream = st;
  // 1. the cos / sin table of every position of the cache
  cfg.gridDim = dim3((unsigned)((s.max_ctx * half + 255) / 256), 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cudaError_t e = cudaLaunchKernelEx(&cfg, rope_table_kernel, s.max_ctx, half, s.hd, (double)rope_base, cs);
  count_launch();
  if (e != cudaSuccess) return e;
  // 2. the rotated queries
  cfg.gridDim = dim3(s.H, a.n_lanes, 1);
  cfg.blockDim = dim3(128, 1, 1);
  e = cudaLaunchKernelEx(&cfg, rope_query_kernel, s, a.iter, a.loops, a.ctx_len, a.h_new, a.Wq, (const float2*)cs, qrot);
  count_launch();
  if (e != cudaSuccess) return e;
  // 3. the scores: K rebuilt on the tensor cores, rotated and dotted in the epilogue (the
  // measurement hook brackets this launch, the call's dominant kernel)
  const int NP = rope_pass_cols(s);
  alignas(64) CUtensorMap tmWk;
  if (!make_tmap_f16(&tmWk, a.Wk, s.d, s.d, s.d, 64, 128)) return cudaErrorInvalidValue;
  const size_t smem = 1024 + 2 * (size_t)kATile + 2 * (size_t)NP * 128 + (size_t)NP * 4;
  int limit = 0;
  if ((e = dyn_smem_limit((const void*)rope_score_kernel, &limit)) != cudaSuccess) return e;
  if (smem > (size_t)limit) return cudaErrorInvalidConfiguration;
  RopeScoreParams p{s, a.iter, a.loops, a.ctx_len, (const uint8_t*)a.codes, (const uint8_t*)a.scales, qrot,
                    (const float2*)cs, scores, reinterpret_cast<uint32_t*>(a.ws + a.wl.status_off), NP};
  cfg.gridDim = dim3((unsigned)((s.max_ctx + 127) / 128), (unsigned)(s.d / NP), (unsigned)a.n_lanes);
  cfg.blockDim = dim3(kRThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  profile_stream_begin(st);
  e = cudaLaunchKernelEx(&cfg, rope_score_kernel, tmWk, p);
  profile_stream_end(st);
  count_launch();
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace tl
