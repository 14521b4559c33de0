// Skinny GEMMs of the decode step on tensor cores (tcgen05, sm_100a), with split-K.
// [Novel Contributions, "Novel Mechanism: Store-h KV Cache": q = W_q h, the absorbed
//  query W_k[j]^T q_j, and the value projection W_v[j] u_j that closes the absorbed form]
//
//   C_part[split][M x N] = A[M x K-range] . B[N x K-range]^T      (fp16 operands, fp32 accumulation)
//
// A is a weight matrix streamed from global memory by TMA in 128 x 64 tiles
// (K-major: rows of W; or MN-major: columns of W, i.e. W^T); B holds the
// batch of activation vectors (lanes, or their fp16 hi/lo halves), N <= 256,
// also K-major, loaded by TMA.  One CTA computes a 128-row block of C over one
// K range; the per-split fp32 partials are reduced in a fixed order by the
// caller's finishing kernel, so results do not depend on scheduling.
//
// Warps: 0 = TMA producer, 1 = MMA issuer / TMEM owner, 2-5 = epilogue
// (TMEM -> registers -> global).  Waits are bounded like in the streaming kernel.
//
// Epilogues (GemmEpi): the absorbed-query GEMM writes the streaming kernel's operand
// image straight from TMEM; the split-K GEMMs (q, out) write fp32 partials and the
// last CTA to finish a 128-row block sums them in split order and writes the result.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "tc_ptx.cuh"
#include "tl_internal.cuh"

namespace tl {
namespace {

using namespace ptx;

constexpr int kStages = 4;
constexpr int kBK = 64;                  // K per stage
constexpr int kABytes = 128 * kBK * 2;   // 16 KB
constexpr long long kGemmWaitLimit = 4000000000ll;

struct GemmParams {
  int M;            // rows of C (multiple of 128)
  int N;            // columns of C (multiple of 16, <= 256)
  int k_per_split;  // multiple of 64
  int a_y_per_z;    // A row offset per blockIdx.z (batched heads)
  int b_y_per_z;    // B row offset per blockIdx.z
  int b_x_per_z;    // B column offset per blockIdx.z
  int a_x_per_z;    // A column offset per blockIdx.z (MN-major A: row offset of W)
  float* out;       // [gridDim.z][splits][M][N] fp32
  uint32_t* status;
};

__device__ __forceinline__ void tma_load_2d_plain(void* dst, const void* tmap, int32_t x, int32_t y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_addr(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(smem_addr(bar))
      : "memory");
}

// A_MN: A given as W^T (MN-major): the tensor map covers W [K rows][M cols]; a stage loads
// two 64 x 64 boxes (M halves).  Otherwise A = W [M rows][K cols], one 128 x 64 box.
// The absorbed-query operand image: row j = fp16(qt_j) and, when the operands are split,
// row 16 + j = fp16(qt_j - fp16(qt_j)); columns in the dequantised position order, 128-byte
// swizzled atom-columns.
__device__ __forceinline__ void put_qimg(const GemmEpiParams& e, int b, int j, int c, float v) {
  const int rows = qimg_rows(e.s.d);
  uint8_t* img = e.qimg + (size_t)b * qimg_bytes(e.s.d);
  const int pos = phys_pos(e.s.fmt, c);
  const __half hi = __float2half_rn(v);
  *reinterpret_cast<__half*>(img + kmajor_offset(j, pos, rows)) = hi;
  if (split_operands(e.s.d))
    *reinterpret_cast<__half*>(img + kmajor_offset(16 + j, pos, rows)) = __float2half_rn(v - __half2float(hi));
}

template <bool A_MN>
__global__ void __launch_bounds__(192, 1) gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA,
                                                         const __grid_constant__ CUtensorMap tmB,
                                                         const GemmParams p, const GemmEpiParams e) {
  const int mblk = blockIdx.x, split = blockIdx.y, z = blockIdx.z;
  const int N = p.N;
  const int nk = p.k_per_split / kBK;
  const int k0 = split * p.k_per_split;
  const uint32_t b_bytes = (uint32_t)N * kBK * 2;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
  uint8_t* sa = base;                            // kStages x 16 KB
  uint8_t* sb = base + kStages * kABytes;        // kStages x (N x 128 B)
  __shared__ uint64_t full[kStages], empty[kStages], done;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  __shared__ int is_last;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(&done, 1);
    abort_flag = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_base;
  volatile int* abort_p = &abort_flag;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nk; ++i, ++issued) {
        const int st = i % kStages, use = i / kStages;
        if (use > 0 && !mbar_wait(&empty[st], (use - 1) & 1, abort_p, kGemmWaitLimit)) break;
        mbar_expect_tx(&full[st], kABytes + b_bytes);
        const int k = k0 + i * kBK;
        if (A_MN) {
          // W rows = K, W columns = M; two 64-column halves of the 128-row block of C
          tma_load_2d_plain(sa + st * kABytes, &tmA, mblk * 128 + z * p.a_x_per_z, k + z * p.a_y_per_z, &full[st]);
          tma_load_2d_plain(sa + st * kABytes + kABytes / 2, &tmA, mblk * 128 + 64 + z * p.a_x_per_z,
                            k + z * p.a_y_per_z, &full[st]);
        } else {
          tma_load_2d_plain(sa + st * kABytes, &tmA, k + z * p.a_x_per_z, mblk * 128 + z * p.a_y_per_z, &full[st]);
        }
        tma_load_2d_plain(sb + st * (N * 128), &tmB, k + z * p.b_x_per_z, z * p.b_y_per_z, &full[st]);
      }
      // loads already issued land before the shared memory goes away
      for (int g = issued > kStages ? issued - kStages : 0; g < issued; ++g) {
        const long long t0 = clock64();
        while (!mbar_try_wait(&full[g % kStages], (g / kStages) & 1) && clock64() - t0 < kGemmWaitLimit) {
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_f16_f32(128, N, A_MN, false);
      const uint64_t a0 = A_MN ? sdesc_sw128(smem_addr(sa), 8192, 1024) : sdesc_sw128(smem_addr(sa), 16, 1024);
      const uint64_t b0 = sdesc_sw128(smem_addr(sb), 16, 1024);
      bool ok = true;
      for (int i = 0; i < nk; ++i) {
        const int st = i % kStages;
        if (!mbar_wait(&full[st], (i / kStages) & 1, abort_p, kGemmWaitLimit)) { ok = false; break; }
        tc_fence_after();
        const uint64_t ad = a0 + (uint64_t)((st * kABytes) >> 4);
        const uint64_t bd = b0 + (uint64_t)((st * N * 128) >> 4);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          // K-major: +32 B per K-step inside the 128-byte atom; MN-major: +16 rows x 128 B
          const uint64_t aoff = A_MN ? (uint64_t)((kk * 2048) >> 4) : (uint64_t)((kk * 32) >> 4);
          if (i == 0 && kk == 0)
            mma_ss_first(tbase, ad + aoff, bd + (uint64_t)((kk * 32) >> 4), idesc);
          else
            mma_ss_acc(tbase, ad + aoff, bd + (uint64_t)((kk * 32) >> 4), idesc);
        }
        mma_commit(&empty[st]);
      }
      mma_commit(&done);
      if (!ok) {
        const long long t0 = clock64();
        while (!mbar_try_wait(&done, 0) && clock64() - t0 < kGemmWaitLimit) {
        }
      }
    }
  } else {
    // epilogue: TMEM lane = row of the 128-row block
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    if (mbar_wait(&done, 0, abort_p, kGemmWaitLimit)) {
      tc_fence_after();
      const uint32_t trow = tbase + ((uint32_t)(quarter * 32) << 16);
      if (e.mode == kEpiQImage) {
        // qt[c][b] = hi column b + lo column nb + b, scaled by log2(e)/sqrt(hd); batch entry z = head
        const int c = mblk * 128 + row;
        const float scale = 1.4426950408889634f / sqrtf((float)e.s.hd);
        for (int b0 = 0; b0 < e.nb; b0 += 16) {
          uint32_t vh[16], vl[16];
          tmem_ld16(trow + b0, vh);
          tmem_ld16(trow + e.nb + b0, vl);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int b = b0 + i;
            int nr;
            if (b < e.n_lanes && lane_active(e.s, e.iter, e.loops, e.ctx_len, b, &nr))
              put_qimg(e, b, z, c, (__uint_as_float(vh[i]) + __uint_as_float(vl[i])) * scale);
          }
        }
        if (z == 0) {
          // the rows of heads j >= H stay zero
          for (int b = 0; b < e.n_lanes; ++b) {
            int nr;
            if (!lane_active(e.s, e.iter, e.loops, e.ctx_len, b, &nr)) continue;
            for (int j = e.s.H; j < kMaxHeads; ++j) put_qimg(e, b, j, c, 0.0f);
          }
        }
      } else {
        float* out = p.out + (((size_t)z * gridDim.y + split) * p.M + (size_t)mblk * 128 + row) * N;
        for (int c = 0; c < N; c += 16) {
          uint32_t v[16];
          tmem_ld16(trow + c, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; i += 4)
            *reinterpret_cast<float4*>(out + c + i) = make_float4(__uint_as_float(v[i]), __uint_as_float(v[i + 1]),
                                                                  __uint_as_float(v[i + 2]), __uint_as_float(v[i + 3]));
        }
        __threadfence();  // the partial is visible device-wide before this CTA is counted
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && abort_flag) atomicOr(p.status, kStatusTimeout);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 256);
  }
  if (e.mode != kEpiQ && e.mode != kEpiOut) return;

  // ---------------------------------------------------------------- split-K reduction by the last CTA
  // Every CTA is counted exactly once (also after a timeout, so the counters stay consistent);
  // the last one of the block resets its counter for the next call.
  if (threadIdx.x == 0) {
    uint32_t* cnt = e.counters + (size_t)z * gridDim.x + mblk;
    const uint32_t old = atomicAdd(cnt, 1u);
    is_last = old == gridDim.y - 1;
    if (is_last) {
      atomicExch(cnt, 0u);
      __threadfence();
    }
  }
  __syncthreads();
  if (!is_last) return;
  const int S = gridDim.y;
  const int nb = e.nb;
  if (e.mode == kEpiQ && mblk == 0 && warp == 0) {
    // range check of the per-lane device values, once per decode call
    for (int b = lane; b < e.n_lanes; b += 32) {
      const int L = e.loops[b], c = e.ctx_len[b];
      if (L < 0 || L > e.s.L_max || c < 0 || c >= e.s.max_ctx) atomicOr(e.status, kStatusRange);
    }
  }
  // items (row, 4 lanes), spread over all threads; the split loads of an item are issued
  // before they are summed (in split order, per component)
  const int items = 128 * (nb / 4);
  for (int it = threadIdx.x; it < items; it += blockDim.x) {
    const int row = it / (nb / 4), b0 = (it % (nb / 4)) * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (e.mode == kEpiQ) {
      const int r = mblk * 128 + row;
      for (int sp0 = 0; sp0 < S; sp0 += 8) {
        float4 t[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (sp0 + k < S) t[k] = __ldcg(reinterpret_cast<const float4*>(p.out + ((size_t)(sp0 + k) * p.M + r) * N + b0));
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (sp0 + k < S) {
            acc.x += t[k].x;
            acc.y += t[k].y;
            acc.z += t[k].z;
            acc.w += t[k].w;
          }
      }
      const float qv[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int b = b0 + i;
        int nr;
        const float q = (b < e.n_lanes && lane_active(e.s, e.iter, e.loops, e.ctx_len, b, &nr)) ? qv[i] : 0.0f;
        const __half hi = __float2half_rn(q);
        e.qhl[(size_t)b * e.s.d + r] = hi;
        e.qhl[(size_t)(nb + b) * e.s.d + r] = __float2half_rn(q - __half2float(hi));
      }
    } else {
      // out feature 128 z + row; with hd = 64 a block holds two heads, whose u columns start at 2 nb
      if (b0 >= e.n_lanes) continue;
      const int c0 = e.s.hd == 64 ? (row >> 6) * 2 * nb : 0;
      for (int sp0 = 0; sp0 < S; sp0 += 8) {
        float4 th[8], tl[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (sp0 + k < S) {
            const float* pr = p.out + (((size_t)z * S + sp0 + k) * 128 + row) * N + c0 + b0;
            th[k] = __ldcg(reinterpret_cast<const float4*>(pr));
            tl[k] = __ldcg(reinterpret_cast<const float4*>(pr + nb));
          }
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (sp0 + k < S) {
            acc.x += th[k].x + tl[k].x;
            acc.y += th[k].y + tl[k].y;
            acc.z += th[k].z + tl[k].z;
            acc.w += th[k].w + tl[k].w;
          }
      }
      const float ov[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int b = b0 + i;
        int nr;
        if (b < e.n_lanes && lane_active(e.s, e.iter, e.loops, e.ctx_len, b, &nr))
          e.out[(size_t)b * e.s.d + (size_t)z * 128 + row] = ov[i];
      }
    }
  }
}


PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

}  // namespace

// fp16 2D tensor map [rows][cols] (row pitch `pitch_elems`), box [box_cols x box_rows], 128-byte swizzle.
bool make_tmap_f16(void* tmap, const void* base, uint64_t rows, uint64_t cols, uint64_t pitch_elems,
                   uint32_t box_cols, uint32_t box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {pitch_elems * 2};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(reinterpret_cast<CUtensorMap*>(tmap), CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims,
             strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_gemm_tc(bool a_mn, const void* tmA, const void* tmB, int M, int N, int K, int splits, int batch,
                           int a_x_per_z, int a_y_per_z, int b_x_per_z, int b_y_per_z, float* out, uint32_t* status,
                           const GemmEpiParams& epi, cudaStream_t st) {
  if (M % 128 || N % 16 || N < 16 || N > 256 || K % (kBK * splits)) return cudaErrorInvalidValue;
  GemmParams p{M, N, K / splits, a_y_per_z, b_y_per_z, b_x_per_z, a_x_per_z, out, status};
  const size_t smem = (size_t)kStages * (kABytes + N * 128) + 1024;
  dim3 grid(M / 128, splits, batch);
  cudaError_t e;
  if (a_mn) {
    e = cudaFuncSetAttribute(gemm_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    gemm_tc_kernel<true><<<grid, 192, smem, st>>>(*reinterpret_cast<const CUtensorMap*>(tmA),
                                                  *reinterpret_cast<const CUtensorMap*>(tmB), p, epi);
  } else {
    e = cudaFuncSetAttribute(gemm_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    gemm_tc_kernel<false><<<grid, 192, smem, st>>>(*reinterpret_cast<const CUtensorMap*>(tmA),
                                                   *reinterpret_cast<const CUtensorMap*>(tmB), p, epi);
  }
  count_launch();
  return cudaGetLastError();
}

}  // namespace tl
