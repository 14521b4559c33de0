/*
 * Seeded synthetic inputs for the store-h decode-attention workloads.
 *
 * This file holds NO arithmetic of the method (no quantiser, no attention, no
 * norm).  It only turns (seed, tensor id, element counter) into numbers:
 *
 *   u64(seed, tid, n)  = fin(key(seed, tid) + n * GAMMA)
 *   key(seed, tid)     = fin(fin(seed + GAMMA) ^ (tid * GAMMA2))
 *
 * where fin() is the SplitMix64 output finaliser and GAMMA its golden-ratio
 * increment (Steele, Lea & Flood, "Fast Splittable Pseudorandom Number
 * Generators", OOPSLA 2014).  Normal deviates use the Box-Muller transform
 * (Box & Muller 1958) in FP64 on the pair of uniforms drawn at counters 2p and
 * 2p+1; element e takes the cosine branch if e is even and the sine branch if
 * e is odd.  FP64 -> binary16 uses round-to-nearest-even (IEEE 754), written
 * out below and checked against numpy's conversion in the tests.
 *
 * Both the CPU oracle's driver and the GPU harness read their inputs from
 * here, so both sides see the same bytes.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GAMMA 0x9E3779B97F4A7C15ull
#define GAMMA2 0xD1B54A32D192ED03ull

static inline uint64_t fin(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

static inline uint64_t key_of(uint64_t seed, uint64_t tid) {
  return fin(fin(seed + GAMMA) ^ (tid * GAMMA2));
}

static inline uint64_t draw(uint64_t key, uint64_t n) { return fin(key + n * GAMMA); }

/* Box-Muller pair p: z[0] (cosine branch) is element 2p, z[1] (sine branch) element 2p+1. */
static inline void normal_pair(uint64_t key, uint64_t p, double z[2]) {
  uint64_t a = draw(key, 2 * p), b = draw(key, 2 * p + 1);
  double u1 = (double)((a >> 11) + 1) * 0x1.0p-53; /* (0, 1] */
  double u2 = (double)(b >> 11) * 0x1.0p-53;       /* [0, 1) */
  double r = sqrt(-2.0 * log(u1));
  double t = 6.283185307179586476925286766559 * u2;
  z[0] = r * cos(t);
  z[1] = r * sin(t);
}

static inline double normal_at(uint64_t key, uint64_t e) {
  double z[2];
  normal_pair(key, e >> 1, z);
  return z[e & 1];
}

/* IEEE binary64 -> binary16, round to nearest, ties to even. */
uint16_t tls_f64_to_f16(double x) {
  uint64_t b;
  memcpy(&b, &x, 8);
  uint16_t sign = (uint16_t)((b >> 48) & 0x8000u);
  uint64_t ab = b & 0x7FFFFFFFFFFFFFFFull;
  if (ab >= 0x7FF0000000000000ull) /* inf or nan */
    return sign | (ab > 0x7FF0000000000000ull ? 0x7E00u : 0x7C00u);
  int bexp = (int)(ab >> 52);
  if (bexp == 0) return sign; /* binary64 subnormal: far below binary16 range */
  int e = bexp - 1023;
  uint64_t m = (ab & 0xFFFFFFFFFFFFFull) | (1ull << 52); /* value = m * 2^(e-52) */
  if (e > 15) return sign | 0x7C00u;
  int shift;
  uint32_t base;
  if (e >= -14) { /* normal binary16: keep 10 fraction bits */
    shift = 42;
    base = (uint32_t)(e + 14) << 10; /* biased exponent minus one, carries absorb the hidden bit */
  } else {        /* subnormal binary16: units of 2^-24 */
    shift = 28 - e;
    base = 0;
    if (shift >= 54) return sign; /* below half of the smallest subnormal */
  }
  uint64_t q = m >> shift;
  uint64_t rem = m & ((1ull << shift) - 1);
  uint64_t half = 1ull << (shift - 1);
  if (rem > half || (rem == half && (q & 1))) q++;
  uint32_t h = base + (uint32_t)q; /* normal: (e+14)<<10 + (1024+frac) = (e+15)<<10 | frac */
  if (h >= 0x7C00u) return sign | 0x7C00u;
  return sign | (uint16_t)h;
}

/* out[i] = f16(scale * N(0,1) at counter offset+i) */
void tls_normal_f16(uint64_t seed, uint64_t tid, uint64_t offset, int64_t n, double scale,
                    uint16_t* out) {
  uint64_t k = key_of(seed, tid);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = tls_f64_to_f16(scale * normal_at(k, offset + (uint64_t)i));
}

/* out[i] = f32(scale * N(0,1) at counter offset+i) */
void tls_normal_f32(uint64_t seed, uint64_t tid, uint64_t offset, int64_t n, double scale,
                    float* out) {
  uint64_t k = key_of(seed, tid);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = (float)(scale * normal_at(k, offset + (uint64_t)i));
}

/* out[i] = normal deviates in FP64 (no rounding), for tests of the generator itself */
void tls_normal_f64(uint64_t seed, uint64_t tid, uint64_t offset, int64_t n, double* out) {
  uint64_t k = key_of(seed, tid);
  for (int64_t i = 0; i < n; ++i) out[i] = normal_at(k, offset + (uint64_t)i);
}

/* out[i] = raw 64-bit draw at counter offset+i */
void tls_u64(uint64_t seed, uint64_t tid, uint64_t offset, int64_t n, uint64_t* out) {
  uint64_t k = key_of(seed, tid);
  for (int64_t i = 0; i < n; ++i) out[i] = draw(k, offset + (uint64_t)i);
}

/*
 * Rows of h: for r in [0, n_rows), row r has row id row_ids[r]; element k of it
 * is N(0,1) at counter row_ids[r]*d + k, times `outlier_mul` if the row's
 * Bernoulli(outlier_p) draw (tensor id `outlier_tid`, counter row_ids[r]) fires.
 * outlier_p <= 0 disables outliers.  Output fp16, row-major [n_rows, d].
 */
/* d must be even. */
void tls_h_rows_f16(uint64_t seed, uint64_t tid, uint64_t outlier_tid, double outlier_p,
                    double outlier_mul, const uint64_t* row_ids, int64_t n_rows, int64_t d,
                    uint16_t* out) {
  uint64_t k = key_of(seed, tid);
  uint64_t ko = key_of(seed, outlier_tid);
  uint64_t thresh = 0;
  if (outlier_p > 0) thresh = (uint64_t)(outlier_p * 18446744073709551616.0);
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < n_rows; ++r) {
    uint64_t rid = row_ids[r];
    double mul = 1.0;
    if (outlier_p > 0 && draw(ko, rid) < thresh) mul = outlier_mul;
    uint16_t* o = out + r * d;
    uint64_t base = rid * (uint64_t)d; /* d is even, so a row holds whole Box-Muller pairs */
    for (int64_t c = 0; c < d; c += 2) {
      double z[2];
      normal_pair(k, (base + (uint64_t)c) >> 1, z);
      o[c] = tls_f64_to_f16(mul * z[0]);
      o[c + 1] = tls_f64_to_f16(mul * z[1]);
    }
  }
}
