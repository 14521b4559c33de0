// Context-streaming kernel of the decode over the iteration-axis delta cache, on 5th-generation
// tensor cores (tcgen05 + TMEM), sm_100a.
// [Architecture-Exclusive Features, "Iteration-axis delta-KV": the state of loop iteration l
//  is rebuilt as h^l = h^0 + sum_{i=1..l} scale_i * dh^i, one FP32 prefix sum per token, in the
//  same kernel that attends the rows]
//
// One CTA = one (lane, split) work item: rows [r_begin, r_end) of lane b, in tiles of 128 rows.
// The dequantisation stage of the store-h decode becomes the FP32 prefix sum: every thread owns
// one row of the tile and rebuilds 32 values at a time from the fp16 anchor and the INT8
// deltas of levels 1..iter (each product code * scale is exact in fp32, each addition rounded
// to fp32, in level order).  The fp32 result x is split into two fp16 operands
// hi = fp16(x), lo = fp16(x - hi), about 22 significant bits together, so the tensor cores see
// the FP32 rebuild rather than an fp16 rounding of it; every MMA is issued once per part into
// the same fp32 accumulators.  The other operands are split the same way at every d_model: the
// absorbed query image has hi and lo rows (qproj writes 32 rows for this call), and P is
// written as hi and lo rows that two N = 16 MMAs accumulate into the same U^T columns.
//
// The absorbed form is that of the store-h decode (k_stream_tc.cu): per head j the scores
// s_cj = qt_j . h_c with the absorbed query image written by qproj_kernel, an online base-2
// softmax, U_j = sum_c p_cj h_c accumulated as U^T in TMEM, and the (m, l, U) partial of the
// split in the workspace layout that oproj_kernel merges.  Per tile:
//   score pass: for each 128-value unit, rebuild -> hi / lo into TMEM -> 2 x 8 TS MMAs into S
//   softmax:    S -> P (fp16 hi / lo), lazy rescale of U^T
//   P.V pass:   for each unit, rebuild again -> hi / lo into shared memory (MN-major) ->
//               4 x 8 SS MMAs (h hi / lo times P hi / lo) into U^T
// The passes run one after the other in all sixteen warps (no warp specialisation): warps w,
// w + 4, w + 8 and w + 12 own the same 32 rows (TMEM lane quarter w) and rebuild one 32-value
// chunk of each unit each; the softmax and the epilogue run in warps 0-3.  The delta cache
// reads (1 + iter) rows per position, and this kernel is written for clarity of the rebuild
// first.  Every wait is bounded; on expiry the kernel records a timeout in the status word,
// waits (bounded) for its MMAs in flight, frees its TMEM and returns.
#include <math_constants.h>

#include "delta_internal.cuh"
#include "tc_ptx.cuh"
#include "tl_internal.cuh"

namespace tl {
namespace {

using namespace ptx;

constexpr int kDSThreads = 512;                 // sixteen warps: four per TMEM lane quarter (32 rows)
constexpr int kStageBytes = 128 * 256;          // one unit of one part, 128 rows x 128 fp16, MN-major
constexpr long long kDWait = 4000000000ll;      // ~2 s of SM clocks

struct DeltaStreamParams {
  DeltaShape s;
  int iter;                     // the real loop iteration: levels 1..iter are summed
  const int32_t* dloops;        // 1 when the lane attends at this call
  const int32_t* ctx_len;
  const __half* anchor;         // [max_lanes][max_ctx][d]
  const int8_t* deltas;         // [L_max-1][max_lanes][max_ctx][d]
  const __half* scales;         // [L_max-1][max_lanes][max_ctx][H]
  const uint8_t* qimg;          // [n_lanes][32 x d] absorbed-query operand images, hi and lo rows
  float* ml;                    // [n_lanes][s_max][16][2]
  float* U;                     // [n_lanes][s_max][16][d]
  uint32_t* status;
  int s_max;
  int split;                    // context rows per split
};

__device__ __forceinline__ uint32_t pack_h2(__half a, __half b) {
  const __half2 h = __halves2half2(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// The FP32 prefix sum of 32 consecutive values [k0, k0 + 32) of one row, split into fp16
// hi / lo pairs (hi[i], lo[i] hold values 2i, 2i+1).  Rows outside the split give zeros.
__device__ __forceinline__ void rebuild32(const DeltaStreamParams& p, size_t row, bool valid, int k0, uint32_t* hi,
                                          uint32_t* lo) {
  const DeltaShape& s = p.s;
  float acc[32];
  if (!valid) {
#pragma unroll
    for (int i = 0; i < 16; ++i) hi[i] = lo[i] = 0u;
    return;
  }
  const uint4* a = reinterpret_cast<const uint4*>(p.anchor + row * s.d + k0);
  uint4 aw[4];
#pragma unroll
  for (int v = 0; v < 4; ++v) aw[v] = __ldg(a + v);
  const size_t level_rows = (size_t)s.max_lanes * s.max_ctx;
  const int head = k0 / s.hd;
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const __half2* h2 = reinterpret_cast<const __half2*>(&aw[v]);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __half22float2(h2[i]);
      acc[8 * v + 2 * i] = f.x;
      acc[8 * v + 2 * i + 1] = f.y;
    }
  }
  uint4 n0 = make_uint4(0, 0, 0, 0), n1 = n0;
  float nsc = 0.0f;
  if (p.iter >= 1) {
    nsc = __half2float(p.scales[row * s.H + head]);
    const uint4* c = reinterpret_cast<const uint4*>(p.deltas + row * s.d + k0);
    n0 = __ldg(c);
    n1 = __ldg(c + 1);
  }
  // level l + 1's loads are issued before level l is added, in level order
  for (int l = 1; l <= p.iter; ++l) {
    const uint4 cw[2] = {n0, n1};
    const float sc = nsc;
    if (l < p.iter) {
      const size_t lr = (size_t)l * level_rows + row;
      nsc = __half2float(p.scales[lr * s.H + head]);
      const uint4* c = reinterpret_cast<const uint4*>(p.deltas + lr * s.d + k0);
      n0 = __ldg(c);
      n1 = __ldg(c + 1);
    }
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      const int8_t* bv = reinterpret_cast<const int8_t*>(&cw[v]);
#pragma unroll
      for (int i = 0; i < 16; ++i) acc[16 * v + i] = __fadd_rn(acc[16 * v + i], __fmul_rn((float)bv[i], sc));
    }
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const __half h0 = __float2half_rn(acc[2 * i]), h1 = __float2half_rn(acc[2 * i + 1]);
    hi[i] = pack_h2(h0, h1);
    lo[i] = pack_h2(__float2half_rn(acc[2 * i] - __half2float(h0)), __float2half_rn(acc[2 * i + 1] - __half2float(h1)));
  }
}

// Bounded wait of all the block's threads on one barrier phase.  The outcome is made
// block-uniform (every thread passes the same __syncthreads sequence afterwards); false on
// expiry anywhere in the block.
__device__ __forceinline__ bool block_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  const bool w = mbar_wait(bar, parity, abort, kDWait);
  return __syncthreads_and(w) != 0;
}

__global__ void __launch_bounds__(kDSThreads, 1) delta_stream_kernel(const DeltaStreamParams p) {
  constexpr int NS = 32;  // query image rows: hi (0-15) and lo (16-31) of each head
  constexpr int NP = 16;  // U^T columns per unit (P hi and lo accumulate into the same ones)
  constexpr int PR = 32;  // P rows: hi (0-15) and lo (16-31)
  constexpr uint32_t kIdS = idesc_f16_f32(128, NS, false, false);
  constexpr uint32_t kIdP = idesc_f16_f32(128, NP, true, false);
  // TMEM columns: S at 0, the score operand's hi / lo staging at 64 / 128, U^T at 256
  constexpr uint32_t kColS = 0, kColHi = 64, kColLo = 128, kColU = 256;
  const DeltaShape& s = p.s;
  const int D = s.d;
  pdl_wait();  // the query images and the new token's rows come from the kernels just before
  const int b = blockIdx.x, split = blockIdx.y;
  if (!p.dloops[b]) return;
  const int n = p.ctx_len[b] + 1;  // < max_ctx + 1: the prep kernel checked ctx_len
  const int r_begin = split * p.split;
  if (r_begin >= n) return;
  const int r_end = min(n, r_begin + p.split);
  const int n_tiles = (r_end - r_begin + 127) >> 7;
  const int n_units = D >> 7;
  const uint32_t qbytes = (uint32_t)(NS * D * 2);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
  uint8_t* qs = base;                        // NS x D fp16, K-major swizzled (the qproj image)
  uint8_t* pv_hi = qs + qbytes;              // one unit, hi part, MN-major
  uint8_t* pv_lo = pv_hi + kStageBytes;      // one unit, lo part
  uint8_t* ps = pv_lo + kStageBytes;         // PR x 128 fp16, K-major swizzled
  __shared__ uint64_t bar_q, bar_mma;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  __shared__ float red[4][16];
  __shared__ float m_sh[16];       // running maximum per head (the same for every row)
  __shared__ float l_sh[16][128];  // running sum per head and tile row

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quarter = warp & 3, grp = warp >> 2;  // grp 0 also runs the softmax and the epilogue
  const int r = quarter * 32 + lane;              // this thread's row of a tile = its TMEM lane
  const int xr = r & 7;
  const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
  for (int i = threadIdx.x; i < 16 * 128; i += kDSThreads) l_sh[i >> 7][i & 127] = 0.0f;
  if (threadIdx.x < 16) m_sh[threadIdx.x] = -CUDART_INF_F;
  if (threadIdx.x == 0) {
    mbar_init(&bar_q, 1);
    mbar_init(&bar_mma, 1);
    abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_base;
  volatile int* abort_p = &abort_flag;
  pdl_trigger();  // TMEM is held

  if (threadIdx.x == 0) {
    mbar_expect_tx(&bar_q, qbytes);
    const uint8_t* src = p.qimg + (size_t)b * qbytes;
    for (uint32_t off = 0; off < qbytes; off += 16384) {
      const uint32_t bytes = min(16384u, qbytes - off);
      asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                       smem_addr(qs + off)),
                   "l"(reinterpret_cast<uint64_t>(src + off)), "r"(bytes), "r"(smem_addr(&bar_q))
                   : "memory");
    }
  }
  bool ok = block_wait(&bar_q, 0, abort_p);
  uint32_t mma_phase = 0;  // completed phases of bar_mma
  bool issued = false;
  // all threads wait for the MMAs committed to bar_mma (one commit per wait)
  auto wait_mma = [&]() -> bool {
    const bool w = block_wait(&bar_mma, mma_phase & 1, abort_p);
    ++mma_phase;
    tc_fence_after();
    return w;
  };

  const uint64_t q_desc0 = sdesc_sw128(smem_addr(qs), 16, 1024);
  const uint64_t hi_desc = sdesc_sw128(smem_addr(pv_hi), 16384, 1024);
  const uint64_t lo_desc = sdesc_sw128(smem_addr(pv_lo), 16384, 1024);
  const uint64_t p_desc = sdesc_sw128(smem_addr(ps), 16, 1024);
  const size_t row_base = (size_t)b * s.max_ctx;

  for (int t = 0; t < n_tiles && ok; ++t) {
    const int row0 = r_begin + t * 128;
    const bool valid = row0 + r < r_end;
    const size_t row = row_base + (size_t)(row0 + r);

    // ---------------------------------------------------------------- score pass
    for (int u = 0; u < n_units && ok; ++u) {
      {
        const int q = grp;  // this warp's 32-value chunk of the unit
        uint32_t hi[16], lo[16];
        rebuild32(p, row, valid, u * 128 + q * 32, hi, lo);
        tmem_st16(tbase + lane_off + kColHi + q * 16, hi);
        tmem_st16(tbase + lane_off + kColLo + q * 16, lo);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncthreads();
      if (warp == 0) {
        tc_fence_after();
        if (elect_one()) {
          const uint64_t bd = q_desc0 + (uint64_t)((u * 2 * NS * 128) >> 4);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint64_t bk = bd + (uint64_t)(((k >> 2) * NS * 128 + (k & 3) * 32) >> 4);
            if (u == 0 && k == 0)
              mma_ts_first(tbase + kColS, tbase + kColHi, bk, kIdS);
            else
              mma_ts_acc(tbase + kColS, tbase + kColHi + k * 8, bk, kIdS);
            mma_ts_acc(tbase + kColS, tbase + kColLo + k * 8, bk, kIdS);
          }
          mma_commit(&bar_mma);
        }
        __syncwarp();
      }
      issued = true;
      ok = wait_mma();  // the staging columns are rewritten by the next unit
    }
    if (!ok) break;

    // ---------------------------------------------------------------- online softmax of the tile
    // warps 0-3 (one thread per row); warps 4-15 only pass the block barriers
    float sc[16], alpha[16], m_new[16];
    bool rescale = false;
    if (grp == 0) {
      uint32_t v[16];
      tmem_ld16(tbase + lane_off + kColS, v);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 16; ++j) sc[j] = __uint_as_float(v[j]);
      tmem_ld16(tbase + lane_off + kColS + 16, v);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 16; ++j) sc[j] += __uint_as_float(v[j]);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (!valid || j >= s.H) sc[j] = -CUDART_INF_F;
        float m = sc[j];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0) red[warp][j] = m;
      }
    }
    __syncthreads();
    if (grp == 0) {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float tm = fmaxf(fmaxf(red[0][j], red[1][j]), fmaxf(red[2][j], red[3][j]));
        const float mu = m_sh[j];
        alpha[j] = 1.0f;
        m_new[j] = mu;
        if (tm > mu + 8.0f) {  // lazy rescale: P stays below 2^8 otherwise
          if (mu != -CUDART_INF_F) {
            alpha[j] = exp2f(mu - tm);
            rescale = true;
          }
          m_new[j] = tm;
        }
      }
    }
    __syncthreads();  // red is reused and m_sh rewritten below
    if (grp == 0) {
      float pr[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        pr[j] = (valid && j < s.H) ? exp2f(sc[j] - m_new[j]) : 0.0f;
        l_sh[j][r] = l_sh[j][r] * alpha[j] + pr[j];
      }
      if (threadIdx.x == 0)
#pragma unroll
        for (int j = 0; j < 16; ++j) m_sh[j] = m_new[j];
      if (__any_sync(0xffffffffu, rescale) && t > 0) {
        // the P.V MMAs of the earlier tiles are complete (each was waited for)
        for (int u = 0; u < n_units; ++u) {
          uint32_t uv[16];
          tmem_ld16(tbase + lane_off + kColU + u * NP, uv);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 16; ++c) uv[c] = __float_as_uint(__uint_as_float(uv[c]) * alpha[c]);
          tmem_st16(tbase + lane_off + kColU + u * NP, uv);
        }
        tmem_st_wait();
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const __half hi = __float2half_rn(pr[j]);
        *reinterpret_cast<__half*>(ps + kmajor_offset(j, r, PR)) = hi;
        *reinterpret_cast<__half*>(ps + kmajor_offset(16 + j, r, PR)) = __float2half_rn(pr[j] - __half2float(hi));
      }
    }

    // ---------------------------------------------------------------- P.V pass
    for (int u = 0; u < n_units && ok; ++u) {
      {
        const int q = grp;  // this warp's 32-value chunk of the unit
        uint32_t hi[16], lo[16];
        rebuild32(p, row, valid, u * 128 + q * 32, hi, lo);
        // values q*32 .. q*32+31 of the unit: atom-column q / 2, 16-byte vectors 4 (q & 1) .. + 3
        const int atom = q >> 1;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const int vv = (q & 1) * 4 + v;
          const uint32_t off = (uint32_t)(atom * 16384 + r * 128 + ((vv ^ xr) << 4));
          *reinterpret_cast<uint4*>(pv_hi + off) = make_uint4(hi[4 * v], hi[4 * v + 1], hi[4 * v + 2], hi[4 * v + 3]);
          *reinterpret_cast<uint4*>(pv_lo + off) = make_uint4(lo[4 * v], lo[4 * v + 1], lo[4 * v + 2], lo[4 * v + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      if (warp == 0) {
        tc_fence_after();
        if (elect_one()) {
          const uint32_t du = tbase + kColU + u * NP;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            // P rows of K-step k: hi at rows 0-15, lo 16 rows (2048 bytes) further
            const uint64_t pk = p_desc + (uint64_t)((((k * 16) >> 6) * PR * 128 + ((k * 16) & 63) * 2) >> 4);
            const uint64_t pl = pk + (uint64_t)(2048 >> 4);
            const uint64_t ah = hi_desc + (uint64_t)((k * 2048) >> 4), al = lo_desc + (uint64_t)((k * 2048) >> 4);
            if (t == 0 && k == 0)
              mma_ss_first(du, ah, pk, kIdP);
            else
              mma_ss_acc(du, ah, pk, kIdP);
            mma_ss_acc(du, ah, pl, kIdP);
            mma_ss_acc(du, al, pk, kIdP);
            mma_ss_acc(du, al, pl, kIdP);
          }
          mma_commit(&bar_mma);
        }
        __syncwarp();
      }
      ok = wait_mma();  // the staging buffers and P are rewritten next
    }
  }

  // ---------------------------------------------------------------- partial (m, l, U) of this split
  if (ok && grp == 0) {
    const size_t part = (size_t)b * p.s_max + split;
    for (int u = 0; u < n_units; ++u) {
      uint32_t uv[16];
      tmem_ld16(tbase + lane_off + kColU + u * NP, uv);
      tmem_ld_wait();
      const int d = u * 128 + r;
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (j < s.H) p.U[(part * kMaxHeads + j) * D + d] = __uint_as_float(uv[j]);
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      float v = l_sh[j][r];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) red[warp][j] = v;
    }
  }
  __syncthreads();
  if (ok && threadIdx.x < 16) {
    const size_t part = (size_t)b * p.s_max + split;
    const int j = threadIdx.x;
    p.ml[(part * kMaxHeads + j) * 2 + 0] = m_sh[j];
    p.ml[(part * kMaxHeads + j) * 2 + 1] = red[0][j] + red[1][j] + red[2][j] + red[3][j];
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && abort_flag) atomicOr(p.status, kStatusTimeout);
  if (warp == 0) {
    if (issued) {
      // nothing may still be writing TMEM when it is freed
      if (elect_one()) mma_commit(&bar_mma);
      __syncwarp();
      const long long t0 = clock64();
      while (!mbar_try_wait(&bar_mma, mma_phase & 1) && clock64() - t0 < kDWait) {
      }
    }
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

cudaError_t launch_kernel(const DeltaStreamParams& p, int n_lanes, cudaStream_t st) {
  const size_t smem = 1024 + 32 * (size_t)p.s.d * 2 + 2 * (size_t)kStageBytes + 32 * 256;
  auto kern = delta_stream_kernel;
  int limit = 0;
  cudaError_t e = dyn_smem_limit((const void*)kern, &limit);
  if (e != cudaSuccess) return e;
  if (smem > (size_t)limit) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_lanes, p.s_max, 1);
  cfg.blockDim = dim3(kDSThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, p);
  count_launch();
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_delta_stream(const DeltaShape& s, const void* anchor, const void* deltas, const void* scales,
                                int iter, int n_lanes, const int32_t* dloops, const int32_t* ctx_len, uint8_t* ws,
                                const Workspace& wl, cudaStream_t st) {
  DeltaStreamParams p{s,
                      iter,
                      dloops,
                      ctx_len,
                      (const __half*)anchor,
                      (const int8_t*)deltas,
                      (const __half*)scales,
                      ws + wl.qt_off,
                      reinterpret_cast<float*>(ws + wl.ml_off),
                      reinterpret_cast<float*>(ws + wl.u_off),
                      reinterpret_cast<uint32_t*>(ws + wl.status_off),
                      wl.s_max,
                      wl.split};
  if (wl.qrows != 32) return cudaErrorInvalidValue;  // the workspace must hold hi / lo query images
  return launch_kernel(p, n_lanes, st);
}

}  // namespace tl
