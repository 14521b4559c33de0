// Context-streaming kernel of store-h decode attention on 5th-generation tensor
// cores (tcgen05 + TMEM), sm_100a.
// [Novel Contributions, "Novel Mechanism: Store-h KV Cache"; Architecture-Exclusive
//  Features, "Store-h KV cache" (FP16-h / INT8-h / INT4-h), "Variable-L KV cache"]
//
// One CTA = one (lane, split) work item: rows [r_begin, r_end) of cache layer
// n_pre+iter of lane b, in tiles of 128 rows.  In the absorbed form, per head j
//   s_cj = qt_j . h_c            (qt = W_k[j]^T q_j, scaled by log2(e)/sqrt(hd))
//   U_j  = sum_c 2^(s_cj - m_j) h_c,   l_j = sum_c 2^(s_cj - m_j)
// Per tile, two tensor-core GEMMs with the tile's dequantised rows H (128 x d):
//   scores  S[128 x N_S]   = H . QT^T   M=128 rows, K=d       A = H from TMEM, B = QT (smem)
//   P.V     U^T[d x N_P]  += H^T . P    M=128 d-values, K=rows A = H (smem, MN-major), B = P (smem)
// U^T accumulates in TMEM over the whole split; the (m, l, U) partial goes to
// the workspace and is merged exactly by the epilogue kernel.
//
// Warp roles (320 threads): warp 0 = TMA producer, warp 1 = MMA issuer (and TMEM
// owner), warps 2-9 = math: two warps per TMEM lane quarter, one for the even and
// one for the odd 128-value units of every row and for heads 0-7 / 8-15 in the
// softmax.  The math warps dequantise each tile twice (into TMEM for the scores,
// into shared memory for P.V, re-reading the codes tile, which is then still in
// L2), run the online softmax in base 2, and write the partial at the end.
// The absorbed query arrives as a ready-made fp16 operand image (written by the
// prologue) through one bulk copy.
//
// Codes tiles arrive through a ring of 16 KB slots (128 rows x 128 bytes,
// 128-byte swizzle) loaded by TMA; every row of a slot is read by its own
// math thread, conflict-free thanks to the swizzle.
//
// Precision: dequantised h is fp16 (INT8 keeps the exact integer codes and
// applies the per-row scale to the scores and to P instead).  When the
// operands fit (d <= 1024), the absorbed query and P are split into fp16
// hi + lo parts (N doubles, which costs nothing at these N), so the scores
// and P.V carry ~22 bits.
//
// INT4 codes are unpacked eight at a time with the magic-number fp16 method
// (OR the nibble into the mantissa of 1024.0 or 64.0, subtract the bias), which
// yields the pairs (e0,e4),(e1,e5),(e2,e6),(e3,e7) of every 32-bit word; the
// d-order inside each group of 8 is therefore permuted, identically for H, QT
// and the rows of U^T, and undone when the partial is written.
//
// Every mbarrier wait is bounded; on expiry the kernel records a timeout in
// the status word, waits (bounded) for its own copies and MMAs in flight,
// frees its TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math_constants.h>

#include <mutex>

#include "tc_ptx.cuh"
#include "tl_internal.cuh"

namespace tl {
namespace {

using namespace ptx;

constexpr int kMathWarps = 8;                  // two per TMEM lane quarter
constexpr int kMathThreads = 32 * kMathWarps;
constexpr int kThreads = 64 + kMathThreads;
constexpr int kRing = 4;                       // codes ring slots
constexpr int kSlotBytes = 128 * 128;          // one ring slot: 128 rows x 128 bytes
constexpr int kPvStageBytes = 128 * 256;       // 128 rows x 128 fp16 values
constexpr int kScaleRowWords = 17;             // 16 words of INT4 group scales (d <= 2048) + 1 of padding
constexpr int kScaleBytes = 2 * 128 * kScaleRowWords * 4;  // one copy per half
constexpr long long kWaitLimit = 4000000000ll; // ~2 s of SM clocks, far beyond any legitimate wait

template <int FMT>
struct Fmt {
  static constexpr int kVals = FMT == TL_H_FP16 ? 64 : FMT == TL_H_INT8_TOKEN ? 128 : 256;  // d-values per 128 B
};

struct StreamParams {
  Shape s;
  int iter;
  const int32_t* loops;
  const int32_t* ctx_len;
  const uint8_t* scales;
  const uint8_t* qimg;  // [n_lanes][qimg_bytes(d)] absorbed-query operand images
  float* ml;            // [n_lanes][s_max][16][2]
  float* U;             // [n_lanes][s_max][16][d]
  uint32_t* status;
  int s_max;
};

struct __align__(8) Bars {
  uint64_t ring_full[kRing], ring_empty[kRing];
  uint64_t stg_full[2], stg_empty[2];
  uint64_t pv_full[2], pv_empty[2];
  uint64_t q_full, s_full, s_empty, p_full, p_empty, u_done, fin;
};

__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 bits_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t* v) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
               : "r"(taddr)
               : "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(v[0]),
               "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_addr(dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_addr(bar))
               : "memory");
}

// Dequantise one 16-byte vector of codes into fp16 pairs.
// FP16: 8 values -> 4 regs; INT8: 16 values -> 8 regs; INT4: 32 values -> 16 regs.
template <int FMT>
__device__ __forceinline__ void dequant_vec(const uint4 v, uint32_t* out, __half2 scale2) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  if (FMT == TL_H_FP16) {
#pragma unroll
    for (int i = 0; i < 4; ++i) out[i] = w[i];
  } else if (FMT == TL_H_INT8_TOKEN) {
    const __half2 bias = __halves2half2(__float2half_rn(1152.0f), __float2half_rn(1152.0f));
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t x = w[i] ^ 0x80808080u;                 // offset binary: code + 128
      const uint32_t a = prmt(x, 0x64646464u, 0x5140u);      // halves 0x64|b0, 0x64|b1 = 1024 + (code + 128)
      const uint32_t b = prmt(x, 0x64646464u, 0x7362u);      // b2, b3
      out[2 * i + 0] = h2_bits(__hsub2(bits_h2(a), bias));
      out[2 * i + 1] = h2_bits(__hsub2(bits_h2(b), bias));
    }
  } else {
    const __half2 bias_lo = __halves2half2(__float2half_rn(1032.0f), __float2half_rn(1032.0f));
    const __half2 bias_hi = __halves2half2(__float2half_rn(72.0f), __float2half_rn(72.0f));
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t x = w[i];
      const uint32_t y = x >> 8;
      // (nibble ^ 8) = code + 8 placed in the mantissa of 1024 (bits 0-3) or 64 (bits 4-7)
      const uint32_t p0 = lop3_and_xor(x, 0x000F000Fu, 0x64086408u);  // (e0, e4)
      const uint32_t p1 = lop3_and_xor(x, 0x00F000F0u, 0x54805480u);  // (e1, e5)
      const uint32_t p2 = lop3_and_xor(y, 0x000F000Fu, 0x64086408u);  // (e2, e6)
      const uint32_t p3 = lop3_and_xor(y, 0x00F000F0u, 0x54805480u);  // (e3, e7)
      out[4 * i + 0] = h2_bits(__hmul2(__hsub2(bits_h2(p0), bias_lo), scale2));
      out[4 * i + 1] = h2_bits(__hmul2(__hsub2(bits_h2(p1), bias_hi), scale2));
      out[4 * i + 2] = h2_bits(__hmul2(__hsub2(bits_h2(p2), bias_lo), scale2));
      out[4 * i + 3] = h2_bits(__hmul2(__hsub2(bits_h2(p3), bias_hi), scale2));
    }
  }
}

template <int FMT, bool SPLIT>
__global__ void __launch_bounds__(kThreads, 1)
    stream_tc_kernel(const __grid_constant__ CUtensorMap tmap, const StreamParams p) {
  constexpr int NS = SPLIT ? 32 : 16;  // score columns (heads, or hi/lo x heads)
  constexpr int NP = SPLIT ? 32 : 16;  // P.V columns
  constexpr int kVals = Fmt<FMT>::kVals;
  constexpr int kRegsPerVec = kVals / 16;  // fp16 pairs per 16-byte code vector
  // ring-slot readers: an INT4 chunk holds two units, one per half; other formats: one half reads it
  constexpr int kSlotReaders = FMT == TL_H_INT4_G64 ? kMathWarps : kMathWarps / 2;
  constexpr int kChunksPerUnit = FMT == TL_H_FP16 ? 2 : 1;
  constexpr int kVecs = FMT == TL_H_INT4_G64 ? 4 : 8;  // vectors of one chunk used by one unit
  constexpr uint32_t kIdS = idesc_f16_f32(128, NS, false, false);
  constexpr uint32_t kIdP = idesc_f16_f32(128, NP, true, false);
  constexpr uint32_t kColS = 0, kColStg = 64, kColU = 256;  // TMEM columns

  const Shape& s = p.s;
  const int D = s.d;
  const int split = blockIdx.x, b = blockIdx.y;
  {
    const int L = p.loops[b], c = p.ctx_len[b];
    if (L < 0 || L > s.L_max || c < 0 || c >= s.max_ctx || p.iter >= L) return;
  }
  const int n = p.ctx_len[b] + 1;
  const int r_begin = split * kSplitRows;
  if (r_begin >= n) return;
  const int r_end = min(n, r_begin + kSplitRows);
  const int n_tiles = (r_end - r_begin + 127) >> 7;
  const int n_units = D >> 7;  // even: d is a multiple of 256
  const int n_chunks = D / kVals;
  const int layer = s.n_pre + p.iter;
  const int row_base = (layer * s.max_lanes + b) * s.max_ctx;
  const uint32_t qbytes = (uint32_t)(NS * D * 2);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
  uint8_t* ring = base;
  uint8_t* qs = ring + kRing * kSlotBytes;    // NS x D fp16, K-major swizzled atom-columns
  uint8_t* pvs = qs + qbytes;                // 2 x [128 rows x 128 fp16]
  uint8_t* ps = pvs + 2 * kPvStageBytes;     // NP x 128 fp16, K-major swizzled
  uint32_t* scs = reinterpret_cast<uint32_t*>(ps + NP * 256);  // INT4: [2][128][17] words of group scales
  __shared__ Bars bars;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  __shared__ float red[2][4][8];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&bars.ring_full[i], 1);
      mbar_init(&bars.ring_empty[i], kSlotReaders);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.stg_full[i], 4);
      mbar_init(&bars.stg_empty[i], 1);
      mbar_init(&bars.pv_full[i], 4);
      mbar_init(&bars.pv_empty[i], 1);
    }
    mbar_init(&bars.q_full, 1);
    mbar_init(&bars.s_full, 1);
    mbar_init(&bars.s_empty, kMathWarps);
    mbar_init(&bars.p_full, kMathWarps);
    mbar_init(&bars.p_empty, 1);
    mbar_init(&bars.u_done, 1);
    mbar_init(&bars.fin, 1);
    abort_flag = 0;
    mbar_fence_init();
    tma_prefetch_desc(&tmap);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_base;
  volatile int* abort_p = &abort_flag;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // the lane's absorbed-query operand image, straight into place
      mbar_expect_tx(&bars.q_full, qbytes);
      const uint8_t* qsrc = p.qimg + (size_t)b * qbytes;
      for (uint32_t off = 0; off < qbytes; off += 16384) bulk_load(qs + off, qsrc + off, 16384, &bars.q_full);
      // first pass over a tile: keep it in L2 for the second (P.V) pass; second pass: last use
      const uint64_t pol_last_use = l2_policy_evict_first();
      const uint64_t pol_keep = l2_policy_evict_normal();
      int issued = 0;
      bool ok = true;
      for (int t = 0; t < n_tiles && ok; ++t) {
        const int gy = row_base + r_begin + t * 128;
        for (int ph = 0; ph < 2 && ok; ++ph) {
          for (int c = 0; c < n_chunks; ++c, ++issued) {
            const int slot = issued & (kRing - 1), use = issued / kRing;
            if (use > 0 && !mbar_wait(&bars.ring_empty[slot], (use - 1) & 1, abort_p, kWaitLimit)) {
              ok = false;
              break;
            }
            mbar_expect_tx(&bars.ring_full[slot], kSlotBytes);
            tma_load_2d(ring + slot * kSlotBytes, &tmap, c * 128, gy, &bars.ring_full[slot],
                        ph == 0 ? pol_keep : pol_last_use);
          }
        }
      }
      {
        // every load issued must land before the CTA's shared memory goes away
        const long long t0 = clock64();
        while (!mbar_try_wait(&bars.q_full, 0) && clock64() - t0 < kWaitLimit) {
        }
      }
      if (!ok) {
        const int first = issued > kRing ? issued - kRing : 0;
        for (int g = first; g < issued; ++g) {
          const long long t0 = clock64();
          while (!mbar_try_wait(&bars.ring_full[g & (kRing - 1)], (g / kRing) & 1) && clock64() - t0 < kWaitLimit) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // base descriptors; the address field is the low 14 bits of (address >> 4), so adding
      // (byte offset >> 4) to a descriptor moves it within shared memory
      const uint64_t q_desc0 = sdesc_sw128(smem_addr(qs), 16, 1024);
      const uint64_t pv_desc0 = sdesc_sw128(smem_addr(pvs), 16384, 1024);
      const uint64_t p_desc0 = sdesc_sw128(smem_addr(ps), 16, 1024);
      bool ok = mbar_wait(&bars.q_full, 0, abort_p, kWaitLimit);
      bool issued_any = false;
      for (int t = 0; t < n_tiles && ok; ++t) {
        if (t > 0 && !mbar_wait(&bars.s_empty, (t - 1) & 1, abort_p, kWaitLimit)) { ok = false; break; }
        for (int u = 0; u < n_units; ++u) {
          const int gs = t * n_units + u, x = u & 1;
          if (!mbar_wait(&bars.stg_full[x], (gs >> 1) & 1, abort_p, kWaitLimit)) { ok = false; break; }
          tc_fence_after();
          // descriptors of this unit's 8 K-steps differ from the first by compile-time byte offsets
          const uint64_t bd = q_desc0 + (uint64_t)((u * 2 * NS * 128) >> 4);
          const uint32_t ta = tbase + kColStg + x * 64;
          if (u == 0)
            mma_ts_first(tbase + kColS, ta, bd, kIdS);
          else
            mma_ts_acc(tbase + kColS, ta, bd, kIdS);
#pragma unroll
          for (int k = 1; k < 8; ++k)
            mma_ts_acc(tbase + kColS, ta + k * 8, bd + (uint64_t)(((k >> 2) * NS * 128 + (k & 3) * 32) >> 4), kIdS);
          issued_any = true;
          mma_commit(&bars.stg_empty[x]);
        }
        if (!ok) break;
        mma_commit(&bars.s_full);
        if (!mbar_wait(&bars.p_full, t & 1, abort_p, kWaitLimit)) { ok = false; break; }
        tc_fence_after();
        for (int u = 0; u < n_units; ++u) {
          const int gp = t * n_units + u, x = u & 1;
          if (!mbar_wait(&bars.pv_full[x], (gp >> 1) & 1, abort_p, kWaitLimit)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad = pv_desc0 + (uint64_t)((x * kPvStageBytes) >> 4);
          const uint32_t du = tbase + kColU + u * NP;
          if (t == 0)
            mma_ss_first(du, ad, p_desc0, kIdP);
          else
            mma_ss_acc(du, ad, p_desc0, kIdP);
#pragma unroll
          for (int k = 1; k < 8; ++k)
            mma_ss_acc(du, ad + (uint64_t)((k * 2048) >> 4),
                       p_desc0 + (uint64_t)((((k * 16) >> 6) * NP * 128 + ((k * 16) & 63) * 2) >> 4), kIdP);
          mma_commit(&bars.pv_empty[x]);
        }
        if (!ok) break;
        mma_commit(&bars.p_empty);
      }
      if (ok) mma_commit(&bars.u_done);
      if (issued_any) {
        // nothing may still be writing TMEM when it is freed
        mma_commit(&bars.fin);
        const long long t0 = clock64();
        while (!mbar_try_wait(&bars.fin, 0) && clock64() - t0 < kWaitLimit) {
        }
      }
    }
  } else {
    // ------------------------------------------------------------ math warps
    // half 0 (warps 2-5) takes the even units and heads 0-7, half 1 (warps 6-9) the odd
    // units and heads 8-15; in each half, warp w owns TMEM lanes / tile rows 32*(w%4) ..
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int h0 = half * 8;  // first head of this half
    uint32_t* sc_row = scs + (half * 128 + r) * kScaleRowWords;
    const uint8_t* my_row = ring + r * 128;
    const int xr = r & 7;

    float m_used[8], l_part[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      m_used[j] = -CUDART_INF_F;
      l_part[j] = 0.0f;
    }
    bool ok = true;

    // scales of a tile's rows (INT8: one fp32; INT4: d/64 fp16, up to 16 words), fetched a tile ahead
    float scale_next = 0.0f;
    uint4 scv_next[4];
    auto fetch_scales = [&](int t_next) {
      const int row0n = r_begin + t_next * 128;
      const bool vn = r < (r_end - row0n);
      const size_t grown = (size_t)row_base + row0n + r;
      if (FMT == TL_H_INT8_TOKEN) scale_next = vn ? reinterpret_cast<const float*>(p.scales)[grown] : 0.0f;
      if (FMT == TL_H_INT4_G64) {
        const uint4* src = reinterpret_cast<const uint4*>(p.scales + grown * (size_t)(D / kInt4Group) * 2);
#pragma unroll
        for (int i = 0; i < 4; ++i) scv_next[i] = (vn && i * 8 < D / kInt4Group) ? src[i] : make_uint4(0, 0, 0, 0);
      }
    };
    fetch_scales(0);

    for (int t = 0; t < n_tiles && ok; ++t) {
      const int row0 = r_begin + t * 128;
      const bool valid = r < (r_end - row0);
      const float scale_row = scale_next;
      if (FMT == TL_H_INT4_G64) {
        // into this thread's own padded smem row (read back one word per unit)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          sc_row[4 * i + 0] = scv_next[i].x;
          sc_row[4 * i + 1] = scv_next[i].y;
          sc_row[4 * i + 2] = scv_next[i].z;
          sc_row[4 * i + 3] = scv_next[i].w;
        }
      }

      for (int ph = 0; ph < 2 && ok; ++ph) {
        if (ph == 1) {
          // ------------------------------------------------ softmax of this tile (this half's heads), then P
          if (!mbar_wait(&bars.s_full, t & 1, abort_p, kWaitLimit)) { ok = false; break; }
          tc_fence_after();
          uint32_t sv[16];
          tmem_ld8(tbase + lane_off + kColS + h0, sv);
          if (NS == 32) tmem_ld8(tbase + lane_off + kColS + 16 + h0, sv + 8);
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars.s_empty);
          float sc[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            float v = __uint_as_float(sv[j]);
            if (NS == 32) v += __uint_as_float(sv[8 + j]);
            if (FMT == TL_H_INT8_TOKEN) v *= scale_row;
            sc[j] = valid ? v : -CUDART_INF_F;
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            float v = sc[j];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
            if (lane == 0) red[half][quarter][j] = v;
          }
          named_bar_sync(1 + half, 128);
          float alpha[8];
          bool rescale = false;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float tm = fmaxf(fmaxf(red[half][0][j], red[half][1][j]), fmaxf(red[half][2][j], red[half][3][j]));
            alpha[j] = 1.0f;
            if (tm > m_used[j] + 8.0f) {  // lazy rescale: P stays below 2^8 otherwise
              if (m_used[j] != -CUDART_INF_F) {
                alpha[j] = exp2f(m_used[j] - tm);
                rescale = true;
              }
              m_used[j] = tm;
            }
          }
          named_bar_sync(1 + half, 128);  // red is rewritten by the next tile
          float pr[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            pr[j] = valid ? exp2f(sc[j] - m_used[j]) : 0.0f;
            l_part[j] = l_part[j] * alpha[j] + pr[j];
          }
          // the previous tile's P.V must be done before P is rewritten or U rescaled
          if (t > 0 && !mbar_wait(&bars.p_empty, (t - 1) & 1, abort_p, kWaitLimit)) { ok = false; break; }
          tc_fence_after();
          if (rescale) {
            // rare: the running maximum rose by more than 2^8; rescale this half's columns of U^T
            for (int u = 0; u < n_units; ++u) {
              uint32_t uv[16];
              tmem_ld8(tbase + lane_off + kColU + u * NP + h0, uv);
              if (NP == 32) tmem_ld8(tbase + lane_off + kColU + u * NP + 16 + h0, uv + 8);
              tmem_ld_wait();
#pragma unroll
              for (int c = 0; c < 16; ++c) uv[c] = __float_as_uint(__uint_as_float(uv[c]) * alpha[c & 7]);
              tmem_st8(tbase + lane_off + kColU + u * NP + h0, uv);
              if (NP == 32) tmem_st8(tbase + lane_off + kColU + u * NP + 16 + h0, uv + 8);
            }
            tmem_st_wait();
          }
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float v = FMT == TL_H_INT8_TOKEN ? pr[j] * scale_row : pr[j];
            const __half hi = __float2half_rn(v);
            *reinterpret_cast<__half*>(ps + kmajor_offset(h0 + j, r, NP)) = hi;
            if (NP == 32)
              *reinterpret_cast<__half*>(ps + kmajor_offset(16 + h0 + j, r, NP)) = __float2half_rn(v - __half2float(hi));
          }
          fence_proxy_async_smem();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars.p_full);
          if (t + 1 < n_tiles) fetch_scales(t + 1);  // lands while this tile's P.V operands are made
        }

        // ------------------------------------------------ dequantise this half's units of the tile
        const int gbase = (t * 2 + ph) * n_chunks;  // producer's load index of chunk 0 of this pass
        for (int u = half; u < n_units && ok; u += 2) {
          uint32_t h[64];
          uint32_t scw = 0;
          if (FMT == TL_H_INT4_G64) scw = sc_row[u];  // fp16 scales of groups 2u (low) and 2u+1 (high)
#pragma unroll
          for (int cc = 0; cc < kChunksPerUnit; ++cc) {
            const int c = FMT == TL_H_INT4_G64 ? (u >> 1) : FMT == TL_H_INT8_TOKEN ? u : 2 * u + cc;
            const int g = gbase + c;
            const int slot = g & (kRing - 1);
            if (!mbar_wait(&bars.ring_full[slot], (g / kRing) & 1, abort_p, kWaitLimit)) { ok = false; break; }
            const uint8_t* src = my_row + slot * kSlotBytes;
            const int v0 = FMT == TL_H_INT4_G64 ? (u & 1) * 4 : 0;
#pragma unroll
            for (int v = 0; v < kVecs; ++v) {
              const uint4 cv = *reinterpret_cast<const uint4*>(src + (((v0 + v) ^ xr) << 4));
              __half2 s2 = __halves2half2(__float2half_rn(1.0f), __float2half_rn(1.0f));
              if (FMT == TL_H_INT4_G64) {
                const uint32_t sbits = (v < 2) ? (scw & 0xFFFFu) : (scw >> 16);
                s2 = bits_h2(sbits | (sbits << 16));
              }
              dequant_vec<FMT>(cv, h + (cc * kVecs + v) * kRegsPerVec, s2);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.ring_empty[slot]);
          }
          if (!ok) break;
          if (!valid) {
#pragma unroll
            for (int i = 0; i < 64; ++i) h[i] = 0u;
          }
          const int gu = t * n_units + u, x = half;
          if (ph == 0) {
            if (gu >= 2 && !mbar_wait(&bars.stg_empty[x], ((gu >> 1) - 1) & 1, abort_p, kWaitLimit)) { ok = false; break; }
            tc_fence_after();
            const uint32_t ta = tbase + lane_off + kColStg + x * 64;
            tmem_st16(ta + 0, h + 0);
            tmem_st16(ta + 16, h + 16);
            tmem_st16(ta + 32, h + 32);
            tmem_st16(ta + 48, h + 48);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.stg_full[x]);
          } else {
            if (gu >= 2 && !mbar_wait(&bars.pv_empty[x], ((gu >> 1) - 1) & 1, abort_p, kWaitLimit)) { ok = false; break; }
            uint8_t* st = pvs + x * kPvStageBytes + r * 128;
#pragma unroll
            for (int v = 0; v < 16; ++v) {
              const uint4 val = make_uint4(h[4 * v], h[4 * v + 1], h[4 * v + 2], h[4 * v + 3]);
              *reinterpret_cast<uint4*>(st + (v >> 3) * 16384 + (((v & 7) ^ xr) << 4)) = val;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.pv_full[x]);
          }
        }
      }
    }

    // ------------------------------------------------ partial (m, l, U) of this split, this half's heads
    if (ok && mbar_wait(&bars.u_done, 0, abort_p, kWaitLimit)) {
      tc_fence_after();
      const size_t part = (size_t)b * p.s_max + split;
      for (int u = 0; u < n_units; ++u) {
        uint32_t uv[16];
        tmem_ld8(tbase + lane_off + kColU + u * NP + h0, uv);
        if (NP == 32) tmem_ld8(tbase + lane_off + kColU + u * NP + 16 + h0, uv + 8);
        tmem_ld_wait();
        const int d = logical_of_pos(FMT, u * 128 + r);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float v = __uint_as_float(uv[j]);
          if (NP == 32) v += __uint_as_float(uv[8 + j]);
          if (h0 + j < s.H) p.U[(part * kMaxHeads + h0 + j) * D + d] = v;
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float v = l_part[j];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) red[half][quarter][j] = v;
      }
      named_bar_sync(1 + half, 128);
      if (r < 8) {
        p.ml[(part * kMaxHeads + h0 + r) * 2 + 0] = m_used[r];
        p.ml[(part * kMaxHeads + h0 + r) * 2 + 1] =
            red[half][0][r] + red[half][1][r] + red[half][2][r] + red[half][3][r];
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && abort_flag) atomicOr(p.status, kStatusTimeout);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// ---------------------------------------------------------------- host side
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

template <int FMT, bool SPLIT>
cudaError_t launch_fmt(const DecodeArgs& a, const CUtensorMap& tmap, cudaStream_t st) {
  const Shape& s = a.s;
  constexpr int NP = SPLIT ? 32 : 16;
  const size_t smem = qimg_bytes(s.d) + 2 * kPvStageBytes + (size_t)NP * 256 + kScaleBytes + 1024 +  // + align
                      (size_t)kRing * kSlotBytes;
  if (smem > 225 * 1024) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(stream_tc_kernel<FMT, SPLIT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  StreamParams p{s,
                 a.iter,
                 a.loops,
                 a.ctx_len,
                 (const uint8_t*)a.scales,
                 a.ws + a.wl.qt_off,
                 reinterpret_cast<float*>(a.ws + a.wl.ml_off),
                 reinterpret_cast<float*>(a.ws + a.wl.u_off),
                 reinterpret_cast<uint32_t*>(a.ws + a.wl.status_off),
                 a.wl.s_max};
  dim3 grid(a.wl.s_max, a.n_lanes);
  stream_tc_kernel<FMT, SPLIT><<<grid, kThreads, smem, st>>>(tmap, p);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_stream(const DecodeArgs& a, cudaStream_t st) {
  const Shape& s = a.s;
  PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap tmap;
  const cuuint64_t dims[2] = {(cuuint64_t)s.row_code_bytes(), (cuuint64_t)s.rows_total()};
  const cuuint64_t strides[1] = {(cuuint64_t)s.row_code_bytes()};
  const cuuint32_t box[2] = {128, 128};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(a.codes), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  const bool split = s.d <= 1024;
  switch (s.fmt) {
    case TL_H_FP16: return split ? launch_fmt<TL_H_FP16, true>(a, tmap, st) : launch_fmt<TL_H_FP16, false>(a, tmap, st);
    case TL_H_INT8_TOKEN:
      return split ? launch_fmt<TL_H_INT8_TOKEN, true>(a, tmap, st) : launch_fmt<TL_H_INT8_TOKEN, false>(a, tmap, st);
    default:
      return split ? launch_fmt<TL_H_INT4_G64, true>(a, tmap, st) : launch_fmt<TL_H_INT4_G64, false>(a, tmap, st);
  }
}

}  // namespace tl
