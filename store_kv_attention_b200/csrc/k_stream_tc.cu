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
// the workspace and is merged exactly by oproj_kernel (k_proj_tc.cu).
//
// Warp roles (640 threads): warp 0 = TMA producer of the score-side ring (and
// the query image); warp 1 = score-MMA issuer (and TMEM owner); warp 2 = P.V-MMA
// issuer; warps 3-10 = score group; warps 11-18 = P.V group; warp 19 = TMA
// producer of the P.V-side ring.  The two groups work on different tiles at the same time:
// while the score group dequantises tile t+1 into TMEM (the A operand of the
// score MMAs) and runs its online softmax, the P.V group dequantises tile t into
// shared memory (the A operand of the P.V MMAs, which take tile t's P).  P is
// double-buffered across tiles; the scores S are double-buffered in TMEM.
// Score group: two warps per TMEM lane quarter, one for the even and one for the
// odd 128-value units of each row, and for heads 0-7 / 8-15 in the softmax.
// P.V group: two warps per 32-row block, one for the even and one for the odd units.
// Each group reads the codes of a tile through its own TMA ring; the second
// read of a tile (P.V) finds it in L2.  The online softmax runs in base 2 and
// each split writes its partial (m, l, U) at the end.
// The absorbed query arrives as a ready-made fp16 operand image (written by
// qproj_kernel) through bulk copies.
//
// Codes tiles arrive in 16 KB slots (128 rows x 128 bytes, 128-byte swizzle)
// loaded by TMA; every row of a slot is read by its own thread, conflict-free
// thanks to the swizzle.  Each ring is split into one sub-ring per set of consumers
// reading the same chunks (so every consumer sees every phase of its slots in order),
// and a slot is released only once the values read from it have been consumed.
//
// The grid is (lane, split) with lanes fastest, so every lane's full-length splits are
// scheduled before any lane's short last split.  The kernel is launched with
// programmatic dependent launch: it waits for qproj_kernel before its first global
// access and lets oproj_kernel be scheduled once it holds its TMEM.
//
// Precision: dequantised h is fp16 (INT8 keeps the exact integer codes and
// applies the per-row scale to the scores and to P instead).  When the
// operands fit (d <= 1024), the absorbed query and P are split into fp16
// hi + lo parts (N doubles, which costs nothing at these N), so the scores
// and P.V carry ~22 bits.
//
// INT4 codes are unpacked eight at a time with the exponent-bias ("magic number")
// integer-to-fp16 conversion -- an identity of IEEE binary16: a small integer n placed in
// the low mantissa bits of the fp16 constant 2^k reads as 2^k + n * ulp(2^k), so one lop3
// (mask, OR the constant, flip the sign bit of the code) and one subtraction give the exact
// value; the method as used for INT4/INT8 weight dequantisation is described by Kim et al.,
// "Who Says Elephants Can't Run" (2022, arXiv:2211.10017).  Here the nibble goes into the
// mantissa of 1024.0 (bits 0-3) or 64.0 (bits 4-7), which
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

#include <algorithm>
#include <mutex>

#include "tc_ptx.cuh"
#include "tl_internal.cuh"

namespace tl {
namespace {

using namespace ptx;

constexpr int kSWarps = 8;                      // score group: two warps per TMEM lane quarter
constexpr int kVWarps = 8;                      // P.V group: two warps per 32-row block
constexpr int kWarpS0 = 3;                      // first score warp
constexpr int kWarpV0 = kWarpS0 + kSWarps;      // first P.V warp
constexpr int kWarpVP = kWarpV0 + kVWarps;     // producer of the P.V-side ring
constexpr int kThreads = 32 * (kWarpVP + 1);
constexpr int kSlotBytes = 128 * 128;           // one ring slot: 128 rows x 128 bytes of codes
constexpr int kPvStageBytes = 128 * 256;        // P.V operand staging: 128 rows x 128 fp16 values
constexpr int kMaxRing = 4;                     // slots per ring at most
constexpr long long kWaitLimit = 4000000000ll;  // ~2 s of SM clocks, far beyond any legitimate wait

template <int FMT>
struct Fmt {
  static constexpr int kVals = FMT == TL_H_FP16 ? 64 : FMT == TL_H_INT8_TOKEN ? 128 : 256;  // d-values per 128 B
  // half-unit (64 values) hh of unit u: ring chunk, first 16-byte vector in it, vectors
  __device__ static int chunk(int u, int hh) {
    return FMT == TL_H_INT4_G64 ? (u >> 1) : FMT == TL_H_INT8_TOKEN ? u : 2 * u + hh;
  }
  __device__ static int vec0(int u, int hh) {
    return FMT == TL_H_INT4_G64 ? (u & 1) * 4 + hh * 2 : FMT == TL_H_INT8_TOKEN ? hh * 4 : 0;
  }
  static constexpr int kVecs = FMT == TL_H_INT4_G64 ? 2 : FMT == TL_H_INT8_TOKEN ? 4 : 8;
  // A score warp reads both halves of its own units: its last read of a chunk is half 1
  // (FP16: every half is a chunk of its own).
  __device__ static bool score_releases(int hh) { return FMT == TL_H_FP16 || hh == 1; }

  // Ring slots.  A consumer waits on a slot's full barrier by phase parity, which is only
  // sound if it sees every use of that slot in order.  So each ring is split into one
  // sub-ring per set of consumers that read the same chunks: INT4 chunks are read by both
  // score halves (and both P.V sets), INT8 chunk g by half / set g & 1, FP16 chunk g by
  // half / set (g >> 1) & 1.
  // Chunk g is the k-th chunk of its owner o and lives in slot o * R + k % R, use k / R,
  // with R the sub-ring size.
  static constexpr int kOwnersS = FMT == TL_H_INT4_G64 ? 1 : 2;
  static constexpr int kOwnersV = kOwnersS;  // the P.V sets read units like the score halves
  __host__ __device__ static void s_slot(int g, int ring, int& slot, int& use) {
    const int R = ring / kOwnersS;
    int o, k;
    if (FMT == TL_H_INT4_G64) {
      o = 0;
      k = g;
    } else if (FMT == TL_H_INT8_TOKEN) {
      o = g & 1;
      k = g >> 1;
    } else {
      o = (g >> 1) & 1;
      k = ((g >> 2) << 1) | (g & 1);
    }
    slot = o * R + k % R;
    use = k / R;
  }
  __host__ __device__ static void v_slot(int g, int ring, int& slot, int& use) { s_slot(g, ring, slot, use); }

  // A consumer warp's place in its sub-ring.  Each consumer warp reads every chunk of its owner
  // (INT4: the one owner; INT8 / FP16: its score half or P.V set) in order, so its k-th chunk
  // is in slot o * R + k % R, use k / R (as s_slot maps it), and the place moves on once per
  // chunk the warp releases -- no division in the consumers' loops.
  struct Cursor {
    int base, R, idx, use;
    __device__ Cursor(int owner, int ring) : base(owner * (ring / kOwnersS)), R(ring / kOwnersS), idx(0), use(0) {}
    __device__ int slot() const { return base + idx; }
    __device__ void next() {
      if (++idx == R) {
        idx = 0;
        ++use;
      }
    }
  };
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
  const LaneSeg* seg;   // rows of each lane (multi-query calls), or NULL: rows 0..ctx_len[b] of lane b
  // Scores given (RoPE variant): fp32 [n_lanes][max_ctx][16], already in the base-2 units of the
  // softmax (and with the INT8 row scale applied).  The score ring and the score MMAs are then
  // not used; NULL = the scores are computed here from the absorbed-query images.
  const float* scores;
  uint32_t* status;
  int s_max;
  int split;            // context rows per split
  int s_ring, v_ring;   // slots of the score-side and P.V-side rings
};

struct __align__(8) Bars {
  uint64_t s_full[kMaxRing], s_empty[kMaxRing];  // score-side codes ring
  uint64_t v_full[kMaxRing], v_empty[kMaxRing];  // P.V-side codes ring
  uint64_t stg_full[2], stg_empty[2];            // TMEM staging of the score A operand, per score half
  uint64_t pv_full[2], pv_empty[2];              // shared-memory staging of the P.V A operand
  uint64_t sc_full[2], sc_empty[2];              // scores S in TMEM, per tile parity
  uint64_t p_full[2], p_empty[2];                // P, per tile parity
  uint64_t red[2];                               // cross-warp reductions of each score half
  uint64_t q_full, u_done, fin_s, fin_v;
};

__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 bits_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }
__device__ __forceinline__ __half2 splat_h(uint32_t bits16) { return bits_h2(bits16 | (bits16 << 16)); }

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
// Bounded wait of a whole warp; the outcome is made warp-uniform.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, kWaitLimit));
}
__device__ __forceinline__ void prefetch_l1(const void* p) {
  asm volatile("prefetch.global.L1 [%0];" ::"l"(reinterpret_cast<uint64_t>(p)));
}
// Bounded wait used only on exit paths: gives up silently after the limit.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity) && clock64() - t0 < kWaitLimit) {
  }
}
// Exit path of a ring producer that issued chunks [0, issued): waits for the latest load into
// each slot.  Only a slot's latest use is waited for: with sub-rings two of the last chunks can
// share a slot, and a barrier that has completed both uses reads as not complete for the older.
// Each owner's latest uses lie within the last 4 x ring chunks.
template <int FMT>
__device__ void drain_ring(uint64_t* full, int ring, int issued) {
  for (int sl = 0; sl < ring; ++sl)
    for (int i = issued - 1; i >= 0 && i >= issued - 4 * ring; --i) {
      int slot, use;
      Fmt<FMT>::s_slot(i, ring, slot, use);
      if (slot == sl) {
        drain_wait(&full[slot], use & 1);
        break;
      }
    }
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
      const uint32_t x = w[i] ^ 0x80808080u;             // offset binary: code + 128
      const uint32_t a = prmt(x, 0x64646464u, 0x5140u);  // halves 0x64|b0, 0x64|b1 = 1024 + (code + 128)
      const uint32_t b = prmt(x, 0x64646464u, 0x7362u);  // b2, b3
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

// INT4: the unit's four 16-byte code vectors of this row (both half-units of unit u lie in one
// slot row), loaded together so that their latencies overlap.
__device__ __forceinline__ void load_unit_int4(const uint8_t* row, int xr, int u, uint4* c) {
  static_assert(2 * Fmt<TL_H_INT4_G64>::kVecs == 4, "an INT4 unit row is four 16-byte vectors");
  const int v0 = (u & 1) * 4;
#pragma unroll
  for (int v = 0; v < 4; ++v) c[v] = *reinterpret_cast<const uint4*>(row + (((v0 + v) ^ xr) << 4));
}
// INT4: half-unit hh of loaded code vectors c into h[32], scale bits from the unit's scale word.
__device__ __forceinline__ void dequant_int4_half(const uint4* c, int hh, uint32_t sw, uint32_t* h) {
  const __half2 s2 = splat_h(hh ? (sw >> 16) : (sw & 0xFFFFu));
  dequant_vec<TL_H_INT4_G64>(c[2 * hh], h, s2);
  dequant_vec<TL_H_INT4_G64>(c[2 * hh + 1], h + 16, s2);
}

// Dequantise half-unit hh (64 values) of unit u from a codes slot row into h[32].
// INT4: the scale of group 2u + hh comes in `sbits` (fp16 bits).
template <int FMT>
__device__ __forceinline__ void dequant_half(const uint8_t* row, int xr, int u, int hh, uint32_t sbits, uint32_t* h) {
  using F = Fmt<FMT>;
  constexpr int kRegsPerVec = F::kVals / 16;
  const __half2 s2 = FMT == TL_H_INT4_G64 ? splat_h(sbits) : __halves2half2(__float2half_rn(1.0f), __float2half_rn(1.0f));
  const int v0 = F::vec0(u, hh);
#pragma unroll
  for (int v = 0; v < F::kVecs; ++v) {
    const uint4 cv = *reinterpret_cast<const uint4*>(row + (((v0 + v) ^ xr) << 4));
    dequant_vec<FMT>(cv, h + v * kRegsPerVec, s2);
  }
}

template <int FMT, bool SPLIT>
__global__ void __launch_bounds__(kThreads, 1)
    stream_tc_kernel(const __grid_constant__ CUtensorMap tmap, const StreamParams p) {
  using F = Fmt<FMT>;
  constexpr int NS = SPLIT ? 32 : 16;  // score columns (heads, or hi/lo x heads)
  constexpr int NP = SPLIT ? 32 : 16;  // P.V columns
  constexpr int kSReaders = FMT == TL_H_INT4_G64 ? kSWarps : kSWarps / 2;  // score warps reading a slot
  constexpr int kVReaders = FMT == TL_H_INT4_G64 ? kVWarps : kVWarps / 2;  // P.V warps reading a slot
  constexpr uint32_t kIdS = idesc_f16_f32(128, NS, false, false);
  constexpr uint32_t kIdP = idesc_f16_f32(128, NP, true, false);
  constexpr uint32_t kColS = 0, kColStg = 64, kColU = 256;  // TMEM columns: S[2] x 32, staging[2] x 64, U^T

  const Shape& s = p.s;
  const int D = s.d;
  pdl_wait();  // the absorbed-query images (and the cache rows) come from the kernels just before
  const int b = blockIdx.x, split = blockIdx.y;
  {
    const int L = p.loops[b], c = p.ctx_len[b];
    if (L < 0 || L > s.L_max || c < 0 || c >= s.max_ctx || p.iter >= L) return;
  }
  // rows of this split: a decode lane's rows 0..ctx_len, or a segment of a multi-query lane
  const LaneSeg g = p.seg ? p.seg[b] : LaneSeg{b, p.ctx_len[b] + 1, 0, 0};
  int r_begin, split_rows;
  if (!seg_split_rows(g, split, p.split, &r_begin, &split_rows)) return;
  const int r_end = r_begin + split_rows;
  const int n_tiles = (r_end - r_begin + 127) >> 7;
  const int n_units = D >> 7;  // even: d is a multiple of 256
  const int n_chunks = D / F::kVals;
  const int layer = s.n_pre + p.iter;
  const int row_base = (layer * s.max_lanes + g.phys) * s.max_ctx;
  const uint32_t qbytes = (uint32_t)(NS * D * 2);
  const int SR = p.s_ring, VR = p.v_ring;
  const int scale_words = D / (2 * kInt4Group);  // INT4: fp16 group scales of a row, two per word

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
  uint8_t* sring = base;                      // SR slots
  uint8_t* vring = sring + SR * kSlotBytes;   // VR slots
  uint8_t* qs = vring + VR * kSlotBytes;      // NS x D fp16, K-major swizzled atom-columns
  uint8_t* pvs = qs + qbytes;                 // 2 x [128 rows x 128 fp16], MN-major swizzled
  uint8_t* ps = pvs + 2 * kPvStageBytes;      // 2 x [NP x 128 fp16], K-major swizzled
  __shared__ Bars bars;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  __shared__ int s_issued;           // score-side chunk loads issued so far
  __shared__ float red[2][2][4][8];  // [parity][score half][quarter][head]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < SR; ++i) {
      mbar_init(&bars.s_full[i], 1);
      mbar_init(&bars.s_empty[i], kSReaders);
    }
    for (int i = 0; i < VR; ++i) {
      mbar_init(&bars.v_full[i], 1);
      mbar_init(&bars.v_empty[i], kVReaders);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.stg_full[i], 4);
      mbar_init(&bars.stg_empty[i], 1);
      mbar_init(&bars.pv_full[i], kVWarps / 2);
      mbar_init(&bars.pv_empty[i], 1);
      mbar_init(&bars.sc_full[i], 1);
      mbar_init(&bars.sc_empty[i], kSWarps);
      mbar_init(&bars.p_full[i], kSWarps);
      mbar_init(&bars.p_empty[i], 1);
      mbar_init(&bars.red[i], 4);
    }
    mbar_init(&bars.q_full, 1);
    mbar_init(&bars.u_done, 1);
    mbar_init(&bars.fin_s, 1);
    mbar_init(&bars.fin_v, 1);
    abort_flag = 0;
    s_issued = 0;
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
  pdl_trigger();  // TMEM is held

  volatile int* s_issued_p = &s_issued;
  const int total_chunks = n_tiles * n_chunks;
  if (warp == 0 && p.scores) {
    // scores given: no score-side loads; the P.V side may load every chunk
    if (lane == 0) *s_issued_p = total_chunks;
  } else if (warp == 0) {
    // ------------------------------------------------------------ TMA producer, score-side ring
    if (lane == 0) {
      // the lane's absorbed-query operand image, straight into place
      mbar_expect_tx(&bars.q_full, qbytes);
      const uint8_t* qsrc = p.qimg + (size_t)b * qbytes;
      for (uint32_t off = 0; off < qbytes; off += 16384)
        bulk_load(qs + off, qsrc + off, min(16384u, qbytes - off), &bars.q_full);
      // the score pass keeps a tile in L2 for the P.V pass, which is its last use
      const uint64_t pol_keep = l2_policy_evict_normal();
      int g = 0;
      for (; g < total_chunks; ++g) {
        int slot, use;
        F::s_slot(g, SR, slot, use);
        if (use > 0 && !mbar_wait(&bars.s_empty[slot], (use - 1) & 1, abort_p, kWaitLimit)) break;
        mbar_expect_tx(&bars.s_full[slot], kSlotBytes);
        tma_load_2d(sring + slot * kSlotBytes, &tmap, (g % n_chunks) * 128, row_base + r_begin + (g / n_chunks) * 128,
                    &bars.s_full[slot], pol_keep);
        *s_issued_p = g + 1;
      }
      // every copy issued lands before the CTA's shared memory goes away
      drain_wait(&bars.q_full, 0);
      drain_ring<FMT>(bars.s_full, SR, g);
    }
  } else if (warp == kWarpVP) {
    // ------------------------------------------------------------ TMA producer, P.V-side ring
    // A chunk's P.V load follows its score load, so it finds the tile in L2.  The score side
    // never waits for this warp's loads of chunks it has not loaded itself, so no cycle forms.
    if (lane == 0) {
      const uint64_t pol_last_use = l2_policy_evict_first();
      int g = 0;
      for (; g < total_chunks; ++g) {
        int slot, use;
        F::v_slot(g, VR, slot, use);
        if (use > 0 && !mbar_wait(&bars.v_empty[slot], (use - 1) & 1, abort_p, kWaitLimit)) break;
        if (*s_issued_p <= g) {
          const long long t0 = clock64();
          while (*s_issued_p <= g && !*abort_p) {
            __nanosleep(128);
            if (clock64() - t0 > kWaitLimit) *abort_p = 1;
          }
          if (*abort_p) break;
        }
        mbar_expect_tx(&bars.v_full[slot], kSlotBytes);
        tma_load_2d(vring + slot * kSlotBytes, &tmap, (g % n_chunks) * 128, row_base + r_begin + (g / n_chunks) * 128,
                    &bars.v_full[slot], pol_last_use);
      }
      drain_ring<FMT>(bars.v_full, VR, g);
    }
  } else if (warp == 1 && p.scores) {
    // scores given: no score MMAs
  } else if (warp == 1) {
    // ------------------------------------------------------------ score-MMA issuer
    // The whole warp runs the loop, so descriptors and TMEM addresses stay warp-uniform, and one
    // elected lane issues (a lone divergent lane issues tcgen05.mma at about half the rate).
    // The address field of a descriptor is (address >> 4), so adding (byte offset >> 4) moves it
    // within shared memory.
    const uint64_t q_desc0 = sdesc_sw128(smem_addr(qs), 16, 1024);
    bool ok = warp_wait(&bars.q_full, 0, abort_p);
    bool issued = false;
    for (int t = 0; t < n_tiles && ok; ++t) {
      const int sb = t & 1;
      if (t >= 2 && !warp_wait(&bars.sc_empty[sb], ((t >> 1) - 1) & 1, abort_p)) { ok = false; break; }
      tc_fence_after();
      const uint32_t dS = tbase + kColS + sb * 32;
      for (int u = 0; u < n_units; ++u) {
        const int x = u & 1, k_use = t * (n_units >> 1) + (u >> 1);
        if (!warp_wait(&bars.stg_full[x], k_use & 1, abort_p)) { ok = false; break; }
        tc_fence_after();
        // the unit's 8 K-steps: A = 8 TMEM columns each, B = 32 bytes within an atom-column
        const uint64_t bd = q_desc0 + (uint64_t)((u * 2 * NS * 128) >> 4);
        const uint32_t ta = tbase + kColStg + x * 64;
        if (elect_one()) {
          if (u == 0)
            mma_ts_first(dS, ta, bd, kIdS);
          else
            mma_ts_acc(dS, ta, bd, kIdS);
#pragma unroll
          for (int k = 1; k < 8; ++k)
            mma_ts_acc(dS, ta + k * 8, bd + (uint64_t)(((k >> 2) * NS * 128 + (k & 3) * 32) >> 4), kIdS);
          mma_commit(&bars.stg_empty[x]);
        }
        __syncwarp();
        issued = true;
      }
      if (!ok) break;
      if (elect_one()) mma_commit(&bars.sc_full[sb]);
      __syncwarp();
    }
    if (issued) {
      // nothing may still be writing TMEM when it is freed
      if (elect_one()) mma_commit(&bars.fin_s);
      __syncwarp();
      drain_wait(&bars.fin_s, 0);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ P.V-MMA issuer (whole warp, one lane issues)
    const uint64_t pv_desc0 = sdesc_sw128(smem_addr(pvs), 16384, 1024);
    const uint64_t p_desc0 = sdesc_sw128(smem_addr(ps), 16, 1024);
    bool ok = true, issued = false;
    for (int t = 0; t < n_tiles && ok; ++t) {
      const int pb = t & 1;
      if (!warp_wait(&bars.p_full[pb], (t >> 1) & 1, abort_p)) { ok = false; break; }
      tc_fence_after();
      const uint64_t pd = p_desc0 + (uint64_t)((pb * NP * 256) >> 4);
      for (int u = 0; u < n_units; ++u) {
        const int x = u & 1, k_use = t * (n_units >> 1) + (u >> 1);
        if (!warp_wait(&bars.pv_full[x], k_use & 1, abort_p)) { ok = false; break; }
        tc_fence_after();
        const uint64_t ad = pv_desc0 + (uint64_t)((x * kPvStageBytes) >> 4);
        const uint32_t du = tbase + kColU + u * NP;
        if (elect_one()) {
          if (t == 0)
            mma_ss_first(du, ad, pd, kIdP);
          else
            mma_ss_acc(du, ad, pd, kIdP);
#pragma unroll
          for (int k = 1; k < 8; ++k)
            mma_ss_acc(du, ad + (uint64_t)((k * 2048) >> 4),
                       pd + (uint64_t)((((k * 16) >> 6) * NP * 128 + ((k * 16) & 63) * 2) >> 4), kIdP);
          mma_commit(&bars.pv_empty[x]);
        }
        __syncwarp();
        issued = true;
      }
      if (!ok) break;
      if (elect_one()) mma_commit(&bars.p_empty[pb]);
      __syncwarp();
    }
    if (ok) {
      if (elect_one()) mma_commit(&bars.u_done);
      __syncwarp();
    }
    if (issued) {
      if (elect_one()) mma_commit(&bars.fin_v);
      __syncwarp();
      drain_wait(&bars.fin_v, 0);
    }
  } else if (warp < kWarpV0) {
    // ------------------------------------------------------------ score group
    // warp -> (TMEM lane quarter = row block, half): half 0 takes the even units and
    // heads 0-7, half 1 the odd units and heads 8-15
    const int quarter = warp & 3;
    const int half = (warp - kWarpS0) >> 2;
    const int r = quarter * 32 + lane;
    const int xr = r & 7;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int h0 = half * 8;
    uint64_t* red_bar = &bars.red[half];

    float m_used[8], l_part[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      m_used[j] = -CUDART_INF_F;
      l_part[j] = 0.0f;
    }
    bool ok = true;
    // per-row scales: INT8 one fp32 (fetched a tile ahead); INT4 d/64 fp16 read per unit,
    // the tile's row brought into L1 a tile ahead
    auto row_of = [&](int t) { return (size_t)row_base + r_begin + t * 128 + r; };
    auto row_valid = [&](int t) { return r < (r_end - (r_begin + t * 128)); };
    float scale_next = 0.0f;
    if (FMT == TL_H_INT8_TOKEN && row_valid(0)) scale_next = __ldg(reinterpret_cast<const float*>(p.scales) + row_of(0));
    if (FMT == TL_H_INT4_G64 && row_valid(0)) prefetch_l1(p.scales + row_of(0) * (size_t)scale_words * 4);

    typename F::Cursor cur(FMT == TL_H_INT4_G64 ? 0 : half, SR);
    for (int t = 0; t < n_tiles && ok; ++t) {
      const bool valid = row_valid(t);
      const float scale_row = scale_next;
      const uint32_t* srow = reinterpret_cast<const uint32_t*>(p.scales + row_of(t) * (size_t)scale_words * 4);
      if (t + 1 < n_tiles && row_valid(t + 1)) {
        if (FMT == TL_H_INT8_TOKEN) scale_next = __ldg(reinterpret_cast<const float*>(p.scales) + row_of(t + 1));
        if (FMT == TL_H_INT4_G64) prefetch_l1(p.scales + row_of(t + 1) * (size_t)scale_words * 4);
      }

      // ------------------------------------------------ this half's units of tile t -> TMEM staging
      // Rows past the lane's end are not zeroed: a score row depends on its own operand row
      // only, and its score is masked to -inf below.
      for (int u = half; u < n_units && !p.scores; u += 2) {
        const uint32_t sw = (FMT == TL_H_INT4_G64 && valid) ? __ldg(srow + u) : 0u;  // groups 2u | 2u+1
        const int k_use = t * (n_units >> 1) + (u >> 1);
        const uint32_t ta = tbase + lane_off + kColStg + half * 64;
        if constexpr (FMT == TL_H_INT4_G64) {
          // one slot wait per unit; the whole unit's codes loaded at once
          const int slot = cur.slot();
          if (!mbar_wait(&bars.s_full[slot], cur.use & 1, abort_p, kWaitLimit)) { ok = false; break; }
          uint4 c[4];
          load_unit_int4(sring + slot * kSlotBytes + r * 128, xr, u, c);
          uint32_t h[32];
          dequant_int4_half(c, 0, sw, h);
          if (k_use >= 1 && !mbar_wait(&bars.stg_empty[half], (k_use - 1) & 1, abort_p, kWaitLimit)) { ok = false; break; }
          tc_fence_after();
          tmem_st16(ta, h);
          tmem_st16(ta + 16, h + 16);
          dequant_int4_half(c, 1, sw, h);
          tmem_st16(ta + 32, h);
          tmem_st16(ta + 48, h + 16);
          // released only after the stores above have taken the values read from the slot
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars.s_empty[slot]);
          cur.next();
        } else {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int slot = cur.slot();
          if (!mbar_wait(&bars.s_full[slot], cur.use & 1, abort_p, kWaitLimit)) { ok = false; break; }
          uint32_t h[32];
          dequant_half<FMT>(sring + slot * kSlotBytes + r * 128, xr, u, hh, hh ? (sw >> 16) : (sw & 0xFFFFu), h);
          if (hh == 0) {
            // the staging buffer is free once the MMAs of this half's previous unit are done
            if (k_use >= 1 && !mbar_wait(&bars.stg_empty[half], (k_use - 1) & 1, abort_p, kWaitLimit)) { ok = false; break; }
            tc_fence_after();
          }
          tmem_st16(ta + hh * 32, h);
          tmem_st16(ta + hh * 32 + 16, h + 16);
          // The slot is released only after the stores above have taken the values read from it:
          // an arrive issued while this warp's shared-memory loads of the slot are still in flight
          // lets the next TMA load into the slot overwrite them before they are read.
          if (F::score_releases(hh)) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.s_empty[slot]);
            cur.next();
          }
        }
        }
        if (!ok) break;
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.stg_full[half]);
      }
      if (!ok) break;

      // ------------------------------------------------ online softmax of tile t, this half's heads
      const int sb = t & 1;
      float sc[8];
      if (p.scores) {
        // scores given: this row's scores of this half's heads (padded heads read as 0)
        const float* srow_s = p.scores + ((size_t)b * s.max_ctx + (r_begin + t * 128 + r)) * kMaxHeads + h0;
#pragma unroll
        for (int j = 0; j < 8; ++j) sc[j] = valid ? (h0 + j < s.H ? srow_s[j] : 0.0f) : -CUDART_INF_F;
      } else {
        if (!mbar_wait(&bars.sc_full[sb], (t >> 1) & 1, abort_p, kWaitLimit)) { ok = false; break; }
        tc_fence_after();
        uint32_t sv[16];
        tmem_ld8(tbase + lane_off + kColS + sb * 32 + h0, sv);
        if (NS == 32) tmem_ld8(tbase + lane_off + kColS + sb * 32 + 16 + h0, sv + 8);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.sc_empty[sb]);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float v = __uint_as_float(sv[j]);
          if (NS == 32) v += __uint_as_float(sv[8 + j]);
          if (FMT == TL_H_INT8_TOKEN) v *= scale_row;
          sc[j] = valid ? v : -CUDART_INF_F;
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float v = sc[j];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0) red[sb][half][quarter][j] = v;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(red_bar);
      if (!mbar_wait(red_bar, t & 1, abort_p, kWaitLimit)) { ok = false; break; }
      float alpha[8];
      bool rescale = false;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float tm = fmaxf(fmaxf(red[sb][half][0][j], red[sb][half][1][j]),
                               fmaxf(red[sb][half][2][j], red[sb][half][3][j]));
        alpha[j] = 1.0f;
        if (tm > m_used[j] + 8.0f) {  // lazy rescale: P stays below 2^8 otherwise
          if (m_used[j] != -CUDART_INF_F) {
            alpha[j] = exp2f(m_used[j] - tm);
            rescale = true;
          }
          m_used[j] = tm;
        }
      }
      float pr[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        pr[j] = valid ? exp2f(sc[j] - m_used[j]) : 0.0f;
        l_part[j] = l_part[j] * alpha[j] + pr[j];
      }
      if (rescale) {
        // rare: the running maximum rose by more than 2^8; U^T is rescaled once every P.V MMA of
        // the earlier tiles has landed (those of tile t wait for this half's P)
        if (t >= 1 && !mbar_wait(&bars.p_empty[(t - 1) & 1], ((t - 1) >> 1) & 1, abort_p, kWaitLimit)) { ok = false; break; }
        tc_fence_after();
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
      // P buffer sb was last read by the P.V MMAs of tile t-2
      if (t >= 2 && !mbar_wait(&bars.p_empty[sb], ((t >> 1) - 1) & 1, abort_p, kWaitLimit)) { ok = false; break; }
      uint8_t* pbuf = ps + sb * NP * 256;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float v = FMT == TL_H_INT8_TOKEN ? pr[j] * scale_row : pr[j];
        const __half hi = __float2half_rn(v);
        *reinterpret_cast<__half*>(pbuf + kmajor_offset(h0 + j, r, NP)) = hi;
        if (NP == 32)
          *reinterpret_cast<__half*>(pbuf + kmajor_offset(16 + h0 + j, r, NP)) = __float2half_rn(v - __half2float(hi));
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars.p_full[sb]);
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
      const int sb = n_tiles & 1;  // last used by tile n_tiles-2, read by every warp since
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float v = l_part[j];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) red[sb][half][quarter][j] = v;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(red_bar);
      if (mbar_wait(red_bar, n_tiles & 1, abort_p, kWaitLimit) && quarter == 0 && lane < 8) {
        float m = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (j == lane) m = m_used[j];
        p.ml[(part * kMaxHeads + h0 + lane) * 2 + 0] = m;
        p.ml[(part * kMaxHeads + h0 + lane) * 2 + 1] =
            red[sb][half][0][lane] + red[sb][half][1][lane] + red[sb][half][2][lane] + red[sb][half][3][lane];
      }
    }
    tmem_st_wait();  // no store of this warp may be in flight when TMEM is freed
  } else {
    // ------------------------------------------------------------ P.V group
    // warp -> (row block, set): set 0 dequantises the even units, set 1 the odd units, each
    // whole unit into its own shared-memory staging buffer that the P.V MMA reads MN-major
    // (d as M, rows as K); a unit's MMAs wait for the four warps of its set only.
    const int vw = warp - kWarpV0;
    const int r = (vw & 3) * 32 + lane;
    const int set = vw >> 2;
    const int xr = r & 7;
    bool ok = true;
    auto row_of = [&](int t) { return (size_t)row_base + r_begin + t * 128 + r; };
    auto row_valid = [&](int t) { return r < (r_end - (r_begin + t * 128)); };
    typename F::Cursor cur(FMT == TL_H_INT4_G64 ? 0 : set, VR);
    for (int t = 0; t < n_tiles && ok; ++t) {
      const bool valid = row_valid(t);
      // Rows past the lane's end meet P = 0.  INT4 rows there get scale 0 and INT8 codes are
      // finite, so only FP16 rows (whose bytes may hold Inf or NaN) are zeroed, and only in a
      // tile that has such rows.
      const bool zero_rows = FMT == TL_H_FP16 && __any_sync(0xffffffffu, !valid);
      const uint32_t* srow = reinterpret_cast<const uint32_t*>(p.scales + row_of(t) * (size_t)scale_words * 4);
      for (int u = set; u < n_units && ok; u += 2) {
        const uint32_t sw = (FMT == TL_H_INT4_G64 && valid) ? __ldg(srow + u) : 0u;  // groups 2u | 2u+1
        const int k_use = t * (n_units >> 1) + (u >> 1);  // this set's units so far
        uint8_t* st = pvs + set * kPvStageBytes + r * 128;
        if constexpr (FMT == TL_H_INT4_G64) {
          const int slot = cur.slot();
          if (!mbar_wait(&bars.v_full[slot], cur.use & 1, abort_p, kWaitLimit)) { ok = false; break; }
          uint4 c[4];
          load_unit_int4(vring + slot * kSlotBytes + r * 128, xr, u, c);
          uint32_t h[32];
          dequant_int4_half(c, 0, sw, h);
          if (k_use >= 1 && !mbar_wait(&bars.pv_empty[set], (k_use - 1) & 1, abort_p, kWaitLimit)) { ok = false; break; }
#pragma unroll
          for (int v = 0; v < 8; ++v)
            *reinterpret_cast<uint4*>(st + ((v ^ xr) << 4)) = make_uint4(h[4 * v], h[4 * v + 1], h[4 * v + 2], h[4 * v + 3]);
          dequant_int4_half(c, 1, sw, h);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            *reinterpret_cast<uint4*>(st + 16384 + ((v ^ xr) << 4)) =
                make_uint4(h[4 * v], h[4 * v + 1], h[4 * v + 2], h[4 * v + 3]);
          // released only after the stores above have taken the values read from the slot
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars.v_empty[slot]);
          cur.next();
        } else {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int slot = cur.slot();
          if (!mbar_wait(&bars.v_full[slot], cur.use & 1, abort_p, kWaitLimit)) { ok = false; break; }
          uint32_t h[32];
          dequant_half<FMT>(vring + slot * kSlotBytes + r * 128, xr, u, hh, hh ? (sw >> 16) : (sw & 0xFFFFu), h);
          if (zero_rows && !valid) {
#pragma unroll
            for (int i = 0; i < 32; ++i) h[i] = 0u;
          }
          // the staging buffer is free once the MMAs of this set's previous unit are done
          if (hh == 0 && k_use >= 1 && !mbar_wait(&bars.pv_empty[set], (k_use - 1) & 1, abort_p, kWaitLimit)) {
            ok = false;
            break;
          }
#pragma unroll
          for (int v = 0; v < 8; ++v)
            *reinterpret_cast<uint4*>(st + hh * 16384 + ((v ^ xr) << 4)) =
                make_uint4(h[4 * v], h[4 * v + 1], h[4 * v + 2], h[4 * v + 3]);
          // released once the stores above have taken the values read from the slot, as on the
          // score side (and with the same reading pattern as a score half)
          if (F::score_releases(hh)) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars.v_empty[slot]);
            cur.next();
          }
        }
        }
        if (!ok) break;
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars.pv_full[set]);
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
  auto kern = stream_tc_kernel<FMT, SPLIT>;
  int limit = 0;
  cudaError_t e = dyn_smem_limit((const void*)kern, &limit);
  if (e != cudaSuccess) return e;
  // fixed regions (+ up to 1 KB of alignment), then as many 16 KB ring slots as fit, shared
  // between the score-side and the P.V-side rings
  const size_t fixed = 1024 + qimg_bytes(s.d) + 2 * (size_t)kPvStageBytes + 2 * (size_t)NP * 256;
  const long long room = (long long)limit - (long long)fixed;
  const int slots = room > 0 ? (int)(room / kSlotBytes) : 0;
  using F = Fmt<FMT>;
  // ring sizes: about half the slots each, multiples of the sub-ring counts
  const int s_ring = std::min(kMaxRing, std::max(F::kOwnersS, (slots + 1) / 2 / F::kOwnersS * F::kOwnersS));
  const int v_ring = std::min(kMaxRing, (slots - s_ring) / F::kOwnersV * F::kOwnersV);
  if (v_ring < F::kOwnersV || v_ring < 2 || s_ring < 2) return cudaErrorInvalidConfiguration;
  const size_t smem = fixed + (size_t)(s_ring + v_ring) * kSlotBytes;
  StreamParams p{s,
                 a.iter,
                 a.loops,
                 a.ctx_len,
                 (const uint8_t*)a.scales,
                 a.ws + a.wl.qt_off,
                 reinterpret_cast<float*>(a.ws + a.wl.ml_off),
                 reinterpret_cast<float*>(a.ws + a.wl.u_off),
                 a.seg,
                 a.scores,
                 reinterpret_cast<uint32_t*>(a.ws + a.wl.status_off),
                 a.wl.s_max,
                 a.wl.split,
                 s_ring,
                 v_ring};
  // lanes vary fastest, so every lane's first splits are scheduled before any lane's last
  // (often short) split, and the full-length CTAs fill the first wave
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.n_lanes, a.wl.s_max, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1] = {pdl_attribute()};
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, tmap, p);
  count_launch();
  if (e != cudaSuccess) return e;
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
