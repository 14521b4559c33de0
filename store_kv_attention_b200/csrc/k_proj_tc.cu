// Fused projections of one decode iteration on tensor cores, one thread-block cluster per
// 128-row block of the projection matrix.
// [Novel Contributions, "Novel Mechanism: Store-h KV Cache": K = W_k h, V = W_v h with the
//  loop block's shared weights, used here in the absorbed form]
//
// qproj (one launch):  q = W_q h_new, then qt_j = W_k[j]^T q_j . log2(e)/sqrt(hd)
//   Cluster mb owns rows [128 mb, 128 mb + 128) of q, i.e. one head (hd = 128) or two
//   (hd = 64).  Rank k of the cluster computes the K-split k of those rows into TMEM; the
//   splits are reduced through distributed shared memory (rank k sums rows of its own
//   share over all ranks, in rank order, into its own copy of the fp16 hi/lo B operand of
//   the second GEMM, then pushes those rows into the other ranks' copies).  The A operand of that GEMM
//   (W_k^T, read MN-major) is loaded by TMA as soon as the first GEMM's operands are dead.
//   Each rank then computes its share of the (head, 128-column block) items of qt and
//   writes the streaming kernel's absorbed-query operand image directly.  With the fused
//   append, each CTA also quantises the new token's row of some lanes into the cache
//   (append_row.cuh) while its first weight tiles load.
//
// oproj (one launch):  u_j = sum_s w_s U_sj (the exact merge of the splits), out_j = W_v[j] u_j
//   Rank k of cluster mb merges the K-slice k of u for the block's heads and every lane into
//   an fp16 hi/lo B operand, multiplies it by its W_v tiles, and the ranks' partial outputs
//   are summed in rank order through distributed shared memory.  The CTAs also run the
//   FP64 safety check, the lanes dealt out over them in turn.
//
// Every reduction runs in a fixed order, so a lane's result does not depend on the
// other lanes of the batch or on scheduling.  All mbarrier waits are bounded; every
// thread reaches both cluster barriers of its kernel whatever happened before them.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math_constants.h>

#include <mutex>

#include "append_row.cuh"
#include "cluster_ptx.cuh"
#include "norm_block.cuh"
#include "tc_ptx.cuh"
#include "tl_internal.cuh"

namespace tl {
namespace {

using namespace ptx;

constexpr int kProjThreads = 128;                // qproj: four warps, TMEM lane quarters 0-3
constexpr int kOProjThreads = 256;               // oproj: eight warps (two per lane quarter)
constexpr int kTileBytes = 128 * 64 * 2;         // one 128 x 64 fp16 operand tile
constexpr long long kProjWaitLimit = 4000000000ll;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return p + ((1024 - (smem_addr(p) & 1023)) & 1023);
}

// The absorbed-query operand image of a lane: row j = fp16(qt_j) and, when the operands
// are split, row 16 + j = fp16(qt_j - fp16(qt_j)); columns in the dequantised position
// order, 128-byte swizzled atom-columns of 64 positions (kmajor_offset).

// Lanes active in this iteration as a 64-bit mask (n_lanes <= 64), computed by warp 0 in
// parallel and broadcast through shared memory; every thread of the block must call it.
__device__ __forceinline__ uint64_t active_mask(const Shape& s, int iter, const int32_t* loops, const int32_t* ctx_len,
                                               int n_lanes, uint64_t* slot) {
  if (threadIdx.x < 32) {
    int nr;
    const int b0 = threadIdx.x, b1 = threadIdx.x + 32;
    const bool a0 = b0 < n_lanes && lane_active(s, iter, loops, ctx_len, b0, &nr);
    const bool a1 = b1 < n_lanes && lane_active(s, iter, loops, ctx_len, b1, &nr);
    const uint32_t lo = __ballot_sync(0xffffffffu, a0), hi = __ballot_sync(0xffffffffu, a1);
    if (threadIdx.x == 0) *slot = (uint64_t)lo | ((uint64_t)hi << 32);
  }
  __syncthreads();
  return *slot;
}

struct QProjParams {
  Shape s;
  int iter;
  const int32_t* loops;
  const int32_t* ctx_len;
  int n_lanes, nb;
  int cl;            // cluster size = K splits of q
  uint32_t* status;
  uint8_t* qimg;     // [n_lanes][qrows x d] fp16
  int qrows;         // 32: fp16 hi + lo rows per head, 16: fp16 rows
  // fused append (codes == NULL: none): h_new of every active lane becomes its new token's row
  const __half* h_new;
  uint8_t* codes;
  uint8_t* scales;
};

// Shared memory: region 0 holds the phase-1 operands; once the phase-1 MMAs are done it
// holds the fp32 partial (read by the other ranks) followed by the phase-2 W_k^T tiles,
// loaded then, and finally the image staging.  Small enough for two CTAs per SM when
// nb <= 32, so all clusters of a launch are resident at once.
struct QProjLayout {
  int KS, nk1, heads_in_block, mblocks, items, ipr, kst2;
  uint32_t part_bytes, region0, a2_bytes, b2_bytes, total;
  uint32_t tmem_cols;  // 128 per phase-2 item (phase 1 uses columns 0..nb-1 first)
  __host__ __device__ QProjLayout(const Shape& s, int nb, int cl) {
    KS = s.d / cl;
    nk1 = KS / 64;
    heads_in_block = 128 / s.hd;
    mblocks = s.d / 128;
    items = heads_in_block * mblocks;
    ipr = (items + cl - 1) / cl;
    kst2 = s.hd / 64;
    const uint32_t ld1 = (uint32_t)nk1 * (kTileBytes + nb * 128);
    const uint32_t stage = 2u * nb * 128u * 2u;             // image staging [hl][nb][128] fp16
    const uint32_t part = 128u * (uint32_t)(nb + 4) * 4u;  // fp32 partial, rows padded by 4 floats
    part_bytes = ((part > stage ? part : stage) + 1023u) & ~1023u;
    a2_bytes = (uint32_t)ipr * kst2 * kTileBytes;
    region0 = ((ld1 > part_bytes + a2_bytes ? ld1 : part_bytes + a2_bytes) + 1023u) & ~1023u;
    b2_bytes = 2u * 2u * nb * 128u;  // two atom-columns of 2 nb rows
    total = 1024u + region0 + b2_bytes;
    tmem_cols = ipr <= 1 ? 128u : ipr <= 2 ? 256u : 512u;
  }
};

__global__ void __launch_bounds__(kProjThreads, 1)
    qproj_kernel(const __grid_constant__ CUtensorMap tmWq, const __grid_constant__ CUtensorMap tmH,
                 const __grid_constant__ CUtensorMap tmWk, const QProjParams p) {
  const Shape& s = p.s;
  const int nb = p.nb, CL = p.cl;
  const QProjLayout lay(s, nb, CL);
  const int k = (int)cluster_rank();  // K split of q; also selects this rank's phase-2 items
  const int mb = blockIdx.y;          // 128-row block of q
  const int it0 = k * lay.ipr, it1 = min(lay.items, it0 + lay.ipr);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = (warp & 3) * 32 + lane;  // TMEM lane of this thread
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align1024(smem_raw);
  uint8_t* a1 = base;                                // nk1 tiles of W_q
  uint8_t* b1 = a1 + lay.nk1 * kTileBytes;           // nk1 tiles of h_new (nb rows)
  float* part = reinterpret_cast<float*>(base);      // after phase-1 MMAs: fp32 partial [128][nb + 4]
  uint8_t* a2 = base + lay.part_bytes;               // phase-2 W_k^T tiles, two 64 x 64 boxes per stage
  uint8_t* b2 = base + lay.region0;                  // q hi/lo operand [2 nb][128], K-major swizzled
  __shared__ uint64_t bar_ld1, bar_ld2, bar_m1, bar_m2;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;

  pdl_wait();  // h_new and the workspace may come from the previous kernel in the stream
  if (threadIdx.x == 0) {
    mbar_init(&bar_ld1, 1);
    mbar_init(&bar_ld2, 1);
    mbar_init(&bar_m1, 1);
    mbar_init(&bar_m2, 1);
    abort_flag = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmWq);
    tma_prefetch_desc(&tmH);
    tma_prefetch_desc(&tmWk);
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base, lay.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_base;
  volatile int* abort_p = &abort_flag;
  pdl_trigger();  // TMEM is held

  // ---------------------------------------------------------------- phase-1 loads (phase 2 loads once they are dead)
  if (threadIdx.x == 0) {
    mbar_expect_tx(&bar_ld1, (uint32_t)lay.nk1 * (kTileBytes + nb * 128));
    for (int i = 0; i < lay.nk1; ++i) {
      const int x = k * lay.KS + 64 * i;
      tma_load_2d(a1 + i * kTileBytes, &tmWq, x, mb * 128, &bar_ld1);
      tma_load_2d(b1 + i * nb * 128, &tmH, x, 0, &bar_ld1);  // rows past n_lanes read as zero
    }
  }

  // ---------------------------------------------------------------- fused append (optional)
  // Each CTA quantises the new token's row of some active lanes into the cache while its weight
  // tiles load.  Nothing in this kernel reads the cache; the streaming kernel that does runs
  // only once this kernel has completed.
  if (p.codes) {
    const int n_ctas = (int)(gridDim.x * gridDim.y);
    for (int b = (int)(blockIdx.y * gridDim.x + blockIdx.x); b < p.n_lanes; b += n_ctas) {
      int nr;
      if (!lane_active(s, p.iter, p.loops, p.ctx_len, b, &nr)) continue;  // the same for the whole CTA
      const size_t row = ((size_t)(s.n_pre + p.iter) * s.max_lanes + b) * s.max_ctx + (size_t)(nr - 1);
      append_row_block<kProjThreads>(s, p.codes, p.scales, row, p.h_new + (size_t)b * s.d);
    }
  }

  // ---------------------------------------------------------------- phase 1: K split k of q
  if (warp == 1) {
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar_ld1, 0, abort_p, kProjWaitLimit));
    if (ok) {
      tc_fence_after();
      if (elect_one()) {
        const uint32_t id1 = idesc_f16_f32(128, nb, false, false);
        for (int i = 0; i < lay.nk1; ++i) {
          const uint64_t ad = sdesc_sw128(smem_addr(a1 + i * kTileBytes), 16, 1024);
          const uint64_t bd = sdesc_sw128(smem_addr(b1 + i * nb * 128), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tbase, ad + (uint64_t)((kk * 32) >> 4), bd + (uint64_t)((kk * 32) >> 4), id1, (i | kk) != 0);
        }
        mma_commit(&bar_m1);
      }
      __syncwarp();
    }
  }
  // partial -> own shared memory (the phase-1 operands are dead once the MMAs are done)
  const int pstride = nb + 4;
  if (mbar_wait(&bar_m1, 0, abort_p, kProjWaitLimit)) {
    tc_fence_after();
    if (threadIdx.x == 0) {
      // the phase-1 operands are dead: load the phase-2 W_k^T tiles behind the partial
      if (it1 > it0) {
        mbar_expect_tx(&bar_ld2, (uint32_t)(it1 - it0) * lay.kst2 * kTileBytes);
        for (int it = it0; it < it1; ++it) {
          const int h2 = it / lay.mblocks, mc = it % lay.mblocks;
          const int j = mb * lay.heads_in_block + h2;
          for (int st = 0; st < lay.kst2; ++st) {
            uint8_t* dst = a2 + ((it - it0) * lay.kst2 + st) * kTileBytes;
            tma_load_2d(dst, &tmWk, mc * 128, j * s.hd + 64 * st, &bar_ld2);
            tma_load_2d(dst + kTileBytes / 2, &tmWk, mc * 128 + 64, j * s.hd + 64 * st, &bar_ld2);
          }
        }
      }
    }
    for (int c0 = 0; c0 < nb; c0 += 16) {
      uint32_t v[16];
      tmem_ld16(tbase + lane_off + c0, v);
      tmem_ld_wait();
      float* dst = part + row * pstride + c0;
#pragma unroll
      for (int i = 0; i < 16; i += 4)
        *reinterpret_cast<float4*>(dst + i) = make_float4(__uint_as_float(v[i]), __uint_as_float(v[i + 1]),
                                                          __uint_as_float(v[i + 2]), __uint_as_float(v[i + 3]));
    }
  }
  tc_fence_before();
  cluster_arrive();  // 1: this rank's partial is in place

  // ---------------------------------------------------------------- reduce the K splits through DSMEM
  // Rank k owns rows [k * 128/CL, (k+1) * 128/CL): it sums them over all ranks in rank order
  // and writes fp16 hi (operand row b) and lo (row nb + b) into every rank's B operand.
  if (mb == 0 && k == 0 && warp == 0) {
    // range check of the per-lane device values, once per decode call
    for (int b = lane; b < p.n_lanes; b += 32) {
      const int L = p.loops[b], c = p.ctx_len[b];
      if (L < 0 || L > s.L_max || c < 0 || c >= s.max_ctx) atomicOr(p.status, kStatusRange);
    }
  }
  __shared__ uint64_t act_slot;
  const uint64_t act = active_mask(s, p.iter, p.loops, p.ctx_len, p.n_lanes, &act_slot);
  const int rpr = 128 / CL;
  cluster_wait();  // 1: every rank's partial is in place
  {
    const int nq = nb / 4;
    const uint32_t part_s = smem_addr(part);
    for (int it = threadIdx.x; it < rpr * nq; it += kProjThreads) {
      const int r = k * rpr + it / nq, b0 = (it % nq) * 4;
      float4 v[8];
#pragma unroll
      for (int rk = 0; rk < 8; ++rk)
        if (rk < CL) v[rk] = dsmem_ld_f4(dsmem_addr(part_s + (uint32_t)((r * pstride + b0) * 4), (uint32_t)rk));
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int rk = 0; rk < 8; ++rk)
        if (rk < CL) {
          acc.x += v[rk].x;
          acc.y += v[rk].y;
          acc.z += v[rk].z;
          acc.w += v[rk].w;
        }
      const float qv[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int b = b0 + i;
        const float q = ((act >> b) & 1) ? qv[i] : 0.0f;
        const __half hi = __float2half_rn(q);
        *reinterpret_cast<__half*>(b2 + kmajor_offset(b, r, 2 * nb)) = hi;
        *reinterpret_cast<__half*>(b2 + kmajor_offset(nb + b, r, 2 * nb)) = __float2half_rn(q - __half2float(hi));
      }
    }
  }
  __syncthreads();  // this rank's rows of the operand are complete in its own copy
  {
    // push them into the other ranks' copies: rows [r0, r0 + rpr) of operand row n are 2 rpr
    // bytes (rpr/8 16-byte chunks) at the same swizzled offsets in every rank's copy
    const uint32_t b2_s = smem_addr(b2);
    const int chunks = rpr / 8;
    const int per_rank = 2 * nb * chunks;
    const int total = (CL - 1) * per_rank;
    for (int it = threadIdx.x; it < total; it += kProjThreads) {
      const int rk = (k + 1 + it / per_rank) % CL;  // every rank but this one
      const int n = (it % per_rank) / chunks, ch = it % chunks;
      const uint32_t off = kmajor_offset(n, k * rpr + ch * 8, 2 * nb);  // 16-byte aligned chunk
      dsmem_st_f4(dsmem_addr(b2_s + off, (uint32_t)rk), *reinterpret_cast<const float4*>(b2 + off));
    }
  }
  fence_proxy_async_smem();
  fence_proxy_async_cluster();
  cluster_sync();  // 2: every rank's operand is complete; no DSMEM access after this point

  // ---------------------------------------------------------------- phase 2: qt = W_k^T q
  // item (h2, mc): head mb * heads_in_block + h2, output columns [128 mc, 128 mc + 128);
  // D of item i at TMEM column 128 i (D of phase 1 is dead by now).
  const bool has_items = it1 > it0;
  if (warp == 1 && has_items) {
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar_ld2, 0, abort_p, kProjWaitLimit));
    if (ok) {
      fence_proxy_async_smem();
      tc_fence_after();
      if (elect_one()) {
        const uint32_t id2 = idesc_f16_f32(128, 2 * nb, true, false);
        for (int it = it0; it < it1; ++it) {
          const int i = it - it0, h2 = it / lay.mblocks;
          for (int st = 0; st < lay.kst2; ++st) {
            const uint64_t ad = sdesc_sw128(smem_addr(a2 + (i * lay.kst2 + st) * kTileBytes), kTileBytes / 2, 1024);
            // K rows [h2 hd + 64 st, +64) of the q block = atom-column h2 kst2 + st of the B operand
            const uint64_t bd = sdesc_sw128(smem_addr(b2 + (h2 * lay.kst2 + st) * 2 * nb * 128), 16, 1024);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss(tbase + 128 * i, ad + (uint64_t)((kk * 2048) >> 4), bd + (uint64_t)((kk * 32) >> 4), id2,
                     (st | kk) != 0);
          }
        }
        mma_commit(&bar_m2);
      }
      __syncwarp();
    }
  }
  // Image epilogue, one item at a time: fp16 hi/lo values are staged in shared memory in the
  // image's physical position order (the dead phase-1 region), then copied out as 16-byte
  // chunks at their swizzled image offsets.  The item loop count is the same for all threads.
  const bool split = p.qrows == 32;
  const int nhl = split ? 2 : 1;
  const int rows_img = p.qrows;
  __half* stg = reinterpret_cast<__half*>(base);  // [hl][nb][128]
  const bool ok2 = has_items && mbar_wait(&bar_m2, 0, abort_p, kProjWaitLimit);
  const float scale = 1.4426950408889634f / sqrtf((float)s.hd);
  for (int it = it0; it < it1; ++it) {
    const int i = it - it0, h2 = it / lay.mblocks, mc = it % lay.mblocks;
    const int j = mb * lay.heads_in_block + h2;
    if (ok2) {
      tc_fence_after();
      const int pp = phys_pos(s.fmt, row);  // blocks are 128-aligned, so the permutation is local
      for (int b0 = 0; b0 < nb; b0 += 16) {
        uint32_t vh[16], vl[16];
        tmem_ld16(tbase + lane_off + 128 * i + b0, vh);
        tmem_ld16(tbase + lane_off + 128 * i + nb + b0, vl);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const float v = (__uint_as_float(vh[q]) + __uint_as_float(vl[q])) * scale;
          const __half hi = __float2half_rn(v);
          stg[(b0 + q) * 128 + pp] = hi;
          if (split) stg[(nb + b0 + q) * 128 + pp] = __float2half_rn(v - __half2float(hi));
        }
      }
    }
    __syncthreads();
    if (ok2) {
      for (int x = threadIdx.x; x < nhl * nb * 16; x += kProjThreads) {
        const int hl = x / (nb * 16), b = (x / 16) % nb, g = x % 16;
        if (!((act >> b) & 1)) continue;
        const uint4 v = *reinterpret_cast<const uint4*>(stg + (hl * nb + b) * 128 + 8 * g);
        uint8_t* img = p.qimg + (size_t)b * rows_img * s.d * 2;
        *reinterpret_cast<uint4*>(img + kmajor_offset(16 * hl + j, mc * 128 + 8 * g, rows_img)) = v;
      }
    }
    __syncthreads();
  }
  if (mb == 0 && s.H < kMaxHeads) {
    // the rows of heads j >= H stay zero; rank k covers columns [k d/CL, (k+1) d/CL)
    const int cs = s.d / CL, groups = cs / 8;
    const int per_lane = (kMaxHeads - s.H) * nhl * groups;
    for (int x = threadIdx.x; x < p.n_lanes * per_lane; x += kProjThreads) {
      const int b = x / per_lane;
      if (!((act >> b) & 1)) continue;
      const int y = x % per_lane;
      const int j = s.H + y / (nhl * groups), hl = (y / groups) % nhl, g = y % groups;
      uint8_t* img = p.qimg + (size_t)b * rows_img * s.d * 2;
      *reinterpret_cast<uint4*>(img + kmajor_offset(16 * hl + j, k * cs + 8 * g, rows_img)) = make_uint4(0, 0, 0, 0);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && abort_flag) atomicOr(p.status, kStatusTimeout);
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, lay.tmem_cols);
  }
}

// ================================================================ oproj
// oproj (one launch): merge the splits of u, out_j = W_v[j] u_j, and the safety check.
//   Cluster mb owns output features [128 mb, 128 mb + 128), i.e. rows of W_v of one head
//   (hd = 128) or two (hd = 64).  Rank k owns the K slice [k KS, (k+1) KS) of u: it merges
//   the streaming kernel's split partials exactly for that slice,
//     u_j = sum_s 2^(m_s - M) U_s / sum_s 2^(m_s - M) l_s   (the same order and operations
//   as a separate merge), writes it as the fp16 hi/lo B operand in shared memory, and
//   multiplies it with its W_v tile (prefetched at kernel start).  The K slices are reduced
//   through DSMEM in rank order, as in qproj.  CTA (k, mb) also runs the per-iteration
//   safety check of lanes mb * CL + k, mb * CL + k + the CTA count, ...
struct OProjParams {
  Shape s;
  int iter;
  const int32_t* loops;
  const int32_t* ctx_len;
  int n_lanes, nb, cl, s_max;
  int split;        // context rows per split
  const float* ml;  // [n_lanes][s_max][16][2]
  const float* U;   // [n_lanes][s_max][16][d]
  const LaneSeg* seg;  // rows of each lane (multi-query calls), or NULL: decode lanes
  float* out;       // [n_lanes][d]
  uint32_t* status;
  const float* residual;
  float threshold;
  uint8_t* flags;
  int32_t* first;
  float* norms;
};

struct OProjLayout {
  int KS, nk, hib, N;
  uint32_t a_bytes, b_bytes, part_bytes, w_bytes, region0, total, tmem_cols;
  __host__ __device__ OProjLayout(const Shape& s, int nb, int cl, int n_lanes, int s_max) {
    KS = s.d / cl;
    nk = KS / 64;
    hib = 128 / s.hd;  // heads in the block
    N = hib * 2 * nb;  // operand rows: per head, nb hi rows then nb lo rows
    a_bytes = (uint32_t)nk * kTileBytes;
    part_bytes = 128u * (uint32_t)(N + 4) * 4u;
    region0 = ((a_bytes > part_bytes ? a_bytes : part_bytes) + 1023u) & ~1023u;
    b_bytes = (uint32_t)N * KS * 2u;
    w_bytes = (((uint32_t)n_lanes * hib * s_max * 4u) + 1023u) & ~1023u;
    total = 1024u + region0 + b_bytes + w_bytes;
    tmem_cols = N <= 32 ? 32u : N <= 64 ? 64u : N <= 128 ? 128u : 256u;
  }
};

__global__ void __launch_bounds__(kOProjThreads, 1)
    oproj_kernel(const __grid_constant__ CUtensorMap tmWv, const OProjParams p) {
  const Shape& s = p.s;
  const int nb = p.nb, CL = p.cl;
  const OProjLayout lay(s, nb, CL, p.n_lanes, p.s_max);
  const int k = (int)cluster_rank();
  const int mb = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = (warp & 3) * 32 + lane;
  const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
  const int N = lay.N;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = align1024(smem_raw);
  uint8_t* a = base;                                   // nk W_v tiles (128 x 64)
  float* part = reinterpret_cast<float*>(base);        // after the MMAs: fp32 partial [128][N + 4]
  uint8_t* bop = base + lay.region0;                   // u hi/lo operand [N][KS], K-major swizzled
  float* wgt = reinterpret_cast<float*>(bop + lay.b_bytes);  // [n_lanes][hib][s_max] merge weights
  __shared__ uint64_t bar_ld, bar_m;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;

  // This kernel is launched (programmatic dependent launch) only once every CTA of the streaming
  // kernel has passed its own griddepcontrol.wait, i.e. once the projection kernel before it has
  // completed, which itself waited for everything enqueued before the decode call.  So the call's
  // inputs -- W_v, loops / ctx_len, the residual, the sticky flags -- are complete here already;
  // only the split partials, written by the streaming kernel, need the wait below.  The weight
  // tiles, the active-lane mask and the safety check therefore overlap the streaming kernel's tail.
  if (threadIdx.x == 0) {
    mbar_init(&bar_ld, 1);
    mbar_init(&bar_m, 1);
    abort_flag = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmWv);
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base, lay.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_base;
  volatile int* abort_p = &abort_flag;

  if (threadIdx.x == 0) {
    mbar_expect_tx(&bar_ld, (uint32_t)lay.nk * kTileBytes);
    for (int i = 0; i < lay.nk; ++i) tma_load_2d(a + i * kTileBytes, &tmWv, k * lay.KS + 64 * i, mb * 128, &bar_ld);
  }

  __shared__ uint64_t act_slot;
  const uint64_t act = active_mask(s, p.iter, p.loops, p.ctx_len, p.n_lanes, &act_slot);
  // the safety check of lanes mb * CL + k, + the CTA count, ... (it depends only on the residual;
  // the trip count and the lane's activity are the same for every thread of the CTA)
  if (p.residual)
    for (int nl = mb * CL + k; nl < p.n_lanes; nl += CL * (int)gridDim.y)
      if ((act >> nl) & 1)
        norm_check_lane<kOProjThreads>(p.residual, nl, s.d, p.threshold, p.iter, p.flags, p.first, p.norms);

  pdl_wait();     // the split partials come from the streaming kernel just before
  pdl_trigger();  // TMEM is held

  // ---------------------------------------------------------------- merge weights
  for (int x = threadIdx.x; x < p.n_lanes * lay.hib; x += kOProjThreads) {
    const int b = x / lay.hib, h2 = x % lay.hib, j = mb * lay.hib + h2;
    if (!((act >> b) & 1)) continue;
    const int S = p.seg ? seg_splits(p.seg[b], p.split) : splits_for_rows(p.ctx_len[b] + 1, p.split);
    const float2* ml = reinterpret_cast<const float2*>(p.ml + (((size_t)b * p.s_max) * kMaxHeads + j) * 2);
    float* wl = wgt + x * p.s_max;
    // (m, l) of the splits, staged in this thread's weight slots before the reductions
    for (int sp = 0; sp < S; ++sp) wl[sp] = 0.0f;
    float M = -CUDART_INF_F;
    for (int sp0 = 0; sp0 < S; sp0 += 8) {
      float2 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (sp0 + u < S) v[u] = ml[(size_t)(sp0 + u) * kMaxHeads];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (sp0 + u < S) {
          M = fmaxf(M, v[u].x);
          wl[sp0 + u] = v[u].x;  // m_s for now
        }
    }
    float L = 0.0f;
    for (int sp = 0; sp < S; ++sp) L += ml[(size_t)sp * kMaxHeads].y * exp2f(wl[sp] - M);
    for (int sp = 0; sp < S; ++sp) wl[sp] = exp2f(wl[sp] - M) / L;
  }
  __syncthreads();

  // ---------------------------------------------------------------- u slice -> B operand
  // item (operand lane b, head h2, 8 consecutive K positions): the hi and lo rows.  Two items
  // per thread at a time, the loads of four splits issued before their multiply-adds, which
  // run in split order.
  {
    const int chunks = lay.KS / 8;
    const int n_items = nb * lay.hib * chunks;
    for (int x0 = threadIdx.x; x0 < n_items; x0 += 2 * kOProjThreads) {
      float v[2][8];
      int S2[2];
      const float* U0[2];
      const float* w2[2];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int x = x0 + q * kOProjThreads;
#pragma unroll
        for (int i = 0; i < 8; ++i) v[q][i] = 0.0f;
        S2[q] = 0;
        U0[q] = nullptr;
        w2[q] = nullptr;
        if (x < n_items) {
          const int b = x / (lay.hib * chunks), h2 = (x / chunks) % lay.hib, ch = x % chunks;
          if (b < p.n_lanes && ((act >> b) & 1)) {
            S2[q] = p.seg ? seg_splits(p.seg[b], p.split) : splits_for_rows(p.ctx_len[b] + 1, p.split);
            U0[q] = p.U + ((size_t)b * p.s_max * kMaxHeads + mb * lay.hib + h2) * s.d + k * lay.KS + 8 * ch;
            w2[q] = wgt + (b * lay.hib + h2) * p.s_max;
          }
        }
      }
      const int Smax = S2[0] > S2[1] ? S2[0] : S2[1];
      for (int sp0 = 0; sp0 < Smax; sp0 += 4) {
        float4 xs[2][8];
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (sp0 + u < S2[q]) {
              const float4* src = reinterpret_cast<const float4*>(U0[q] + (size_t)(sp0 + u) * kMaxHeads * s.d);
              xs[q][2 * u] = __ldcs(src);
              xs[q][2 * u + 1] = __ldcs(src + 1);
            }
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (sp0 + u < S2[q]) {
              const float ws = w2[q][sp0 + u];
              v[q][0] = fmaf(ws, xs[q][2 * u].x, v[q][0]);
              v[q][1] = fmaf(ws, xs[q][2 * u].y, v[q][1]);
              v[q][2] = fmaf(ws, xs[q][2 * u].z, v[q][2]);
              v[q][3] = fmaf(ws, xs[q][2 * u].w, v[q][3]);
              v[q][4] = fmaf(ws, xs[q][2 * u + 1].x, v[q][4]);
              v[q][5] = fmaf(ws, xs[q][2 * u + 1].y, v[q][5]);
              v[q][6] = fmaf(ws, xs[q][2 * u + 1].z, v[q][6]);
              v[q][7] = fmaf(ws, xs[q][2 * u + 1].w, v[q][7]);
            }
      }
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int x = x0 + q * kOProjThreads;
        if (x >= n_items) continue;
        const int b = x / (lay.hib * chunks), h2 = (x / chunks) % lay.hib, ch = x % chunks;
        __align__(16) __half hi[8], lo[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          hi[i] = __float2half_rn(v[q][i]);
          lo[i] = __float2half_rn(v[q][i] - __half2float(hi[i]));
        }
        const int nh = h2 * 2 * nb + b, nlo = h2 * 2 * nb + nb + b;
        *reinterpret_cast<uint4*>(bop + kmajor_offset(nh, 8 * ch, N)) = *reinterpret_cast<const uint4*>(hi);
        *reinterpret_cast<uint4*>(bop + kmajor_offset(nlo, 8 * ch, N)) = *reinterpret_cast<const uint4*>(lo);
      }
    }
  }
  fence_proxy_async_smem();
  __syncthreads();

  // ---------------------------------------------------------------- out partial of K slice k
  if (warp == 1) {
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar_ld, 0, abort_p, kProjWaitLimit));
    if (ok) {
      tc_fence_after();
      if (elect_one()) {
        const uint32_t id = idesc_f16_f32(128, N, false, false);
        for (int i = 0; i < lay.nk; ++i) {
          const uint64_t ad = sdesc_sw128(smem_addr(a + i * kTileBytes), 16, 1024);
          const uint64_t bd = sdesc_sw128(smem_addr(bop + i * N * 128), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss(tbase, ad + (uint64_t)((kk * 32) >> 4), bd + (uint64_t)((kk * 32) >> 4), id, (i | kk) != 0);
        }
        mma_commit(&bar_m);
      }
      __syncwarp();
    }
  }
  const int pstride = N + 4;
  if (mbar_wait(&bar_m, 0, abort_p, kProjWaitLimit)) {
    tc_fence_after();
    // warps w and w + 4 share lane quarter w % 4 and take alternate 16-column groups
    for (int c0 = (warp >> 2) * 16; c0 < N; c0 += 32) {
      uint32_t v[16];
      tmem_ld16(tbase + lane_off + c0, v);
      tmem_ld_wait();
      float* dst = part + row * pstride + c0;
#pragma unroll
      for (int i = 0; i < 16; i += 4)
        *reinterpret_cast<float4*>(dst + i) = make_float4(__uint_as_float(v[i]), __uint_as_float(v[i + 1]),
                                                          __uint_as_float(v[i + 2]), __uint_as_float(v[i + 3]));
    }
  }
  tc_fence_before();
  cluster_sync();  // 1: every rank's partial is in place

  // ---------------------------------------------------------------- reduce the K slices, write out
  // rank k: rows [k * 128/CL, (k+1) * 128/CL) of the block, 4 lanes per item; per rank the hi
  // and lo columns of a lane are added, then the ranks are summed in rank order
  {
    const int rpr = 128 / CL, nq = nb / 4;
    const uint32_t part_s = smem_addr(part);
    for (int x = threadIdx.x; x < rpr * nq; x += kOProjThreads) {
      const int r = k * rpr + x / nq, b0 = (x % nq) * 4;
      if (b0 >= p.n_lanes) continue;
      const int c0 = (r / s.hd) * 2 * nb;  // the head's columns in the operand
      float4 vh[8], vl[8];
#pragma unroll
      for (int rk = 0; rk < 8; ++rk)
        if (rk < CL) {
          vh[rk] = dsmem_ld_f4(dsmem_addr(part_s + (uint32_t)((r * pstride + c0 + b0) * 4), (uint32_t)rk));
          vl[rk] = dsmem_ld_f4(dsmem_addr(part_s + (uint32_t)((r * pstride + c0 + nb + b0) * 4), (uint32_t)rk));
        }
      float o[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int rk = 0; rk < 8; ++rk)
        if (rk < CL) {
          o[0] += vh[rk].x + vl[rk].x;
          o[1] += vh[rk].y + vl[rk].y;
          o[2] += vh[rk].z + vl[rk].z;
          o[3] += vh[rk].w + vl[rk].w;
        }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int b = b0 + i;
        if (b < p.n_lanes && ((act >> b) & 1)) p.out[(size_t)b * s.d + (size_t)mb * 128 + r] = o[i];
      }
    }
  }
  cluster_arrive();  // 2: this rank reads no other rank's partial any more

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && abort_flag) atomicOr(p.status, kStatusTimeout);
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, lay.tmem_cols);
  }
  cluster_wait();  // 2: no rank leaves while its partial may still be read
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

// Cluster size of the projection kernels: the largest power of two up to 8 that divides d / 64,
// so that every K slice (d / CL) is a whole number of 64-value tiles and every rank's share of
// the 128 rows of a block (128 / CL) is a whole number of 8-row groups.
int proj_cluster(int d) {
  int cl = 8;
  while (cl > 1 && (d / 64) % cl != 0) cl >>= 1;
  return cl;
}

// Dynamic shared memory oproj_kernel needs for a call (its merge weights grow with the splits).
size_t oproj_smem_bytes(const Shape& s, int n_lanes, int s_max) {
  return OProjLayout(s, lanes_padded(n_lanes), proj_cluster(s.d), n_lanes, s_max).total;
}

cudaError_t launch_qproj(const DecodeArgs& a, cudaStream_t st) {
  const Shape& s = a.s;
  const Workspace& w = a.wl;
  const int CL = proj_cluster(s.d);
  const QProjLayout lay(s, w.nb, CL);
  alignas(64) CUtensorMap tmWq, tmH, tmWk;
  if (!make_tmap_f16(&tmWq, a.Wq, s.d, s.d, s.d, 64, 128) || !make_tmap_f16(&tmH, a.h_new, a.n_lanes, s.d, s.d, 64, w.nb) ||
      !make_tmap_f16(&tmWk, a.Wk, s.d, s.d, s.d, 64, 64))
    return cudaErrorInvalidValue;
  int limit = 0;
  cudaError_t e = dyn_smem_limit((const void*)qproj_kernel, &limit);
  if (e != cudaSuccess) return e;
  if (lay.total > (uint32_t)limit) return cudaErrorInvalidConfiguration;
  QProjParams p{s,
                a.iter,
                a.loops,
                a.ctx_len,
                a.n_lanes,
                w.nb,
                CL,
                reinterpret_cast<uint32_t*>(a.ws + w.status_off),
                a.ws + w.qt_off,
                w.qrows,
                a.h_new,
                a.append ? (uint8_t*)a.codes : nullptr,
                a.append ? (uint8_t*)a.scales : nullptr};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CL, s.d / 128, 1);
  cfg.blockDim = dim3(kProjThreads, 1, 1);
  cfg.dynamicSmemBytes = lay.total;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1] = pdl_attribute();
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, qproj_kernel, tmWq, tmH, tmWk, p);
  count_launch();
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_oproj(const DecodeArgs& a, cudaStream_t st) {
  const Shape& s = a.s;
  const Workspace& w = a.wl;
  const int CL = proj_cluster(s.d);
  const OProjLayout lay(s, w.nb, CL, a.n_lanes, w.s_max);
  alignas(64) CUtensorMap tmWv;
  if (!make_tmap_f16(&tmWv, a.Wv, s.d, s.d, s.d, 64, 128)) return cudaErrorInvalidValue;
  int limit = 0;
  cudaError_t e = dyn_smem_limit((const void*)oproj_kernel, &limit);
  if (e != cudaSuccess) return e;
  if (lay.total > (uint32_t)limit) return cudaErrorInvalidConfiguration;
  OProjParams p{s,
                a.iter,
                a.loops,
                a.ctx_len,
                a.n_lanes,
                w.nb,
                CL,
                w.s_max,
                w.split,
                reinterpret_cast<const float*>(a.ws + w.ml_off),
                reinterpret_cast<const float*>(a.ws + w.u_off),
                a.seg,
                a.out,
                reinterpret_cast<uint32_t*>(a.ws + w.status_off),
                a.residual,
                a.threshold,
                a.abort_flags,
                a.first_abort_iter,
                a.norms};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CL, s.d / 128, 1);
  cfg.blockDim = dim3(kOProjThreads, 1, 1);
  cfg.dynamicSmemBytes = lay.total;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1] = pdl_attribute();
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, oproj_kernel, tmWv, p);
  count_launch();
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace tl
