// Plain, slow CPU oracle of the store-h decode-attention path, in C++ with FP64 arithmetic.
//
// TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's CPU-baseline
// leg load this library (through oracle/cpp.py); the CUDA library never does, and the two
// share no code, header or table.  Every function is written as the definition it follows,
// in the order the pages give, with plain loops: no blocking, no reordering beyond the
// definition, so that it can be checked against the pages by eye.
//
// What it computes, and where the pages define it:
//   * Store-h cache: the cache keeps the pre-QKV hidden state h of every (layer, token);
//     attention rebuilds K = W_k h and V = W_v h with the loop block's shared weights.
//     [Novel Contributions, "Novel Mechanism: Store-h KV Cache";
//      Architecture-Exclusive Features, "Store-h KV cache"]
//   * Storage modes FP16-h / INT8-h / INT4-h [same section, mode table]; the pages give only
//     byte counts, so the quantisers follow the workload statement: INT8 symmetric per token,
//     scale = amax/127 (fp32); INT4 symmetric per group of 64 along d, scale = fp16(amax/7);
//     round half to even; two codes per byte, low nibble first.  Dequantisation is exact.
//   * Per-iteration safety check on the L2 norm of the FP32 residual, strict "exceeds".
//     [Novel Contributions, "Novel: Per-Iteration Safety Check"]
// Readings where the pages are silent: softmax scale 1/sqrt(head_dim), no positional
// rotation and no biases, the new token's query from its unquantised fp16 h.
//
// Build: g++ -O2 -std=c++17 -fopenmp -fPIC -shared -ffp-contract=off (no fast-math: fp32
// divisions and rounding stay IEEE).
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

// ---------------------------------------------------------------- IEEE binary16 <-> binary64 / binary32
// binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
double f16_to_f64(uint16_t h) {
  const int sign = h >> 15;
  const int e = (h >> 10) & 0x1F;
  const int f = h & 0x3FF;
  double v;
  if (e == 0)
    v = ldexp((double)f, -24);  // subnormal: f * 2^-24
  else if (e == 31)
    v = f ? NAN : INFINITY;
  else
    v = ldexp((double)(1024 + f), e - 25);  // (1 + f/1024) * 2^(e-15)
  return sign ? -v : v;
}

// Round a binary32 value to the nearest binary16, ties to even (IEEE 754 roundTiesToEven).
uint16_t f32_to_f16_rne(float x) {
  uint32_t u;
  memcpy(&u, &x, 4);
  const uint16_t sign = (uint16_t)((u >> 16) & 0x8000);
  const double a = fabs((double)x);  // exact
  if (isnan(x)) return (uint16_t)(sign | 0x7E00);
  if (a >= 65520.0) return (uint16_t)(sign | 0x7C00);  // rounds to infinity (65504 + half an ulp of 32)
  // the spacing of binary16 values near a: 2^(E-10) for normals with exponent E >= -14, 2^-24 below
  int E;
  frexp(a, &E);  // a = m * 2^E, m in [0.5, 1)  =>  floor(log2 a) = E - 1
  int exp2 = E - 1;
  if (exp2 < -14) exp2 = -14;
  const double ulp = ldexp(1.0, exp2 - 10);
  const double q = a / ulp;  // exact: a has at most 24 significant bits
  double n = floor(q);
  const double rem = q - n;
  if (rem > 0.5 || (rem == 0.5 && fmod(n, 2.0) != 0.0)) n += 1.0;
  const double r = n * ulp;  // the rounded magnitude
  if (r >= 65520.0) return (uint16_t)(sign | 0x7C00);
  // encode r
  if (r < ldexp(1.0, -14)) return (uint16_t)(sign | (uint16_t)(r / ldexp(1.0, -24)));  // subnormal or zero
  int Er;
  const double mr = frexp(r, &Er);  // r = mr * 2^Er
  const int e16 = Er - 1 + 15;
  const int frac = (int)((mr * 2.0 - 1.0) * 1024.0);
  return (uint16_t)(sign | (uint16_t)(e16 << 10) | (uint16_t)frac);
}

float f16_to_f32(uint16_t h) { return (float)f16_to_f64(h); }

}  // namespace

extern "C" {

// ---------------------------------------------------------------- quantiser (the write side)
// h: fp16 bits [n][d].  fmt 0: codes = the fp16 bytes; 1: int8 codes [n][d] + fp32 scale [n];
// 2: int4 codes [n][d/2] + fp16 scale bits [n][d/64].
void oracle_quantize_rows(int fmt, int d, int64_t n, const uint16_t* h, uint8_t* codes, void* scales) {
  for (int64_t i = 0; i < n; ++i) {
    const uint16_t* x = h + i * d;
    if (fmt == 0) {
      memcpy(codes + i * 2 * d, x, 2 * (size_t)d);
    } else if (fmt == 1) {
      // INT8 per token: amax = max |x| (exact in fp32), scale = amax / 127 (fp32 division),
      // code = clamp(rne(x / scale), -127, 127) with an fp32 quotient; zero scale -> zero codes
      float amax = 0.0f;
      for (int k = 0; k < d; ++k) {
        const float v = fabsf(f16_to_f32(x[k]));
        if (v > amax) amax = v;
      }
      const float scale = amax / 127.0f;
      ((float*)scales)[i] = scale;
      int8_t* c = (int8_t*)(codes + i * d);
      for (int k = 0; k < d; ++k) {
        if (scale > 0.0f) {
          const float q = f16_to_f32(x[k]) / scale;
          float r = nearbyintf(q);  // default rounding mode: to nearest, ties to even
          if (r > 127.0f) r = 127.0f;
          if (r < -127.0f) r = -127.0f;
          c[k] = (int8_t)r;
        } else {
          c[k] = 0;
        }
      }
    } else {
      // INT4 per group of 64: scale = fp16_rne(amax / 7.0f), code = clamp(rne(x / float(scale)), -7, 7),
      // byte j of a group = code[2j] & 0xF | (code[2j+1] & 0xF) << 4
      const int G = d / 64;
      uint16_t* sc = (uint16_t*)scales + i * G;
      uint8_t* c = codes + i * (d / 2);
      for (int g = 0; g < G; ++g) {
        float amax = 0.0f;
        for (int k = 0; k < 64; ++k) {
          const float v = fabsf(f16_to_f32(x[g * 64 + k]));
          if (v > amax) amax = v;
        }
        const uint16_t s16 = f32_to_f16_rne(amax / 7.0f);
        sc[g] = s16;
        const float div = f16_to_f32(s16);
        int8_t code[64];
        for (int k = 0; k < 64; ++k) {
          if (div > 0.0f) {
            float r = nearbyintf(f16_to_f32(x[g * 64 + k]) / div);
            if (r > 7.0f) r = 7.0f;
            if (r < -7.0f) r = -7.0f;
            code[k] = (int8_t)r;
          } else {
            code[k] = 0;
          }
        }
        for (int j = 0; j < 32; ++j)
          c[g * 32 + j] = (uint8_t)((code[2 * j] & 0xF) | ((code[2 * j + 1] & 0xF) << 4));
      }
    }
  }
}

// Exact dequantisation into FP64: h_hat = code * scale (fp16 rows as they are).
void oracle_dequantize_rows(int fmt, int d, int64_t n, const uint8_t* codes, const void* scales, double* out) {
  for (int64_t i = 0; i < n; ++i) {
    double* o = out + i * d;
    if (fmt == 0) {
      const uint16_t* x = (const uint16_t*)(codes + i * 2 * d);
      for (int k = 0; k < d; ++k) o[k] = f16_to_f64(x[k]);
    } else if (fmt == 1) {
      const int8_t* c = (const int8_t*)(codes + i * d);
      const double s = (double)((const float*)scales)[i];
      for (int k = 0; k < d; ++k) o[k] = (double)c[k] * s;
    } else {
      const uint8_t* c = codes + i * (d / 2);
      const uint16_t* sc = (const uint16_t*)scales + i * (d / 64);
      for (int k = 0; k < d; ++k) {
        const int nib = (k & 1) ? (c[k / 2] >> 4) : (c[k / 2] & 0xF);
        const int code = nib >= 8 ? nib - 16 : nib;  // two's complement nibble
        o[k] = (double)code * f16_to_f64(sc[k / 64]);
      }
    }
  }
}

// ---------------------------------------------------------------- attention of one head
// Rows j*hd .. j*hd+hd-1 of an fp16 [out][in] weight, as FP64 (exact).
static std::vector<double> head_rows(const uint16_t* W, int j, int d, int hd) {
  std::vector<double> w((size_t)hd * d);
  for (int r = 0; r < hd; ++r)
    for (int k = 0; k < d; ++k) w[(size_t)r * d + k] = f16_to_f64(W[(size_t)(j * hd + r) * d + k]);
  return w;
}

// The definition, with K and V rebuilt explicitly: for head j (rows j*hd .. j*hd+hd-1 of the
// [out][in] weights), q_j = W_q[j] h_new, K_cj = W_k[j] h_c, V_cj = W_v[j] h_c for every row c,
// s_c = q_j . K_cj / sqrt(hd), p = softmax(s), o_j = sum_c p_c V_cj.
static void attend_head_explicit(int j, int64_t n, int d, int hd, const double* h_hat, const uint16_t* h_new,
                                 const uint16_t* Wq, const uint16_t* Wk, const uint16_t* Wv, double* out_j) {
  // the head's weight rows in FP64 (exact), converted once
  std::vector<double> wq = head_rows(Wq, j, d, hd), wk = head_rows(Wk, j, d, hd), wv = head_rows(Wv, j, d, hd);
  std::vector<double> hn(d), q(hd), s(n), K(hd), V((size_t)n * hd);
  for (int k = 0; k < d; ++k) hn[k] = f16_to_f64(h_new[k]);
  for (int r = 0; r < hd; ++r) {
    double acc = 0.0;
    for (int k = 0; k < d; ++k) acc += wq[(size_t)r * d + k] * hn[k];
    q[r] = acc;
  }
  const double inv = 1.0 / sqrt((double)hd);
  for (int64_t c = 0; c < n; ++c) {
    const double* h = h_hat + c * d;
    for (int r = 0; r < hd; ++r) {
      const double* rk = &wk[(size_t)r * d];
      const double* rv = &wv[(size_t)r * d];
      double ak = 0.0, av = 0.0;
      for (int k = 0; k < d; ++k) {
        ak += rk[k] * h[k];
        av += rv[k] * h[k];
      }
      K[r] = ak;
      V[(size_t)c * hd + r] = av;
    }
    double dot = 0.0;
    for (int r = 0; r < hd; ++r) dot += q[r] * K[r];
    s[c] = dot * inv;
  }
  double m = -INFINITY;
  for (int64_t c = 0; c < n; ++c)
    if (s[c] > m) m = s[c];
  double Z = 0.0;
  for (int64_t c = 0; c < n; ++c) {
    s[c] = exp(s[c] - m);
    Z += s[c];
  }
  for (int r = 0; r < hd; ++r) out_j[r] = 0.0;
  for (int64_t c = 0; c < n; ++c) {
    const double p = s[c] / Z;
    for (int r = 0; r < hd; ++r) out_j[r] += p * V[(size_t)c * hd + r];
  }
}

// The algebraically equal absorbed form, for lanes too long for the explicit rebuild on a CPU:
// qt_j = W_k[j]^T q_j, s_c = qt_j . h_c / sqrt(hd), p = softmax(s), u_j = sum_c p_c h_c,
// o_j = W_v[j] u_j.
static void attend_head_absorbed(int j, int64_t n, int d, int hd, const double* h_hat, const uint16_t* h_new,
                                 const uint16_t* Wq, const uint16_t* Wk, const uint16_t* Wv, double* out_j) {
  std::vector<double> wq = head_rows(Wq, j, d, hd), wk = head_rows(Wk, j, d, hd), wv = head_rows(Wv, j, d, hd);
  std::vector<double> hn(d), q(hd), qt(d, 0.0), s(n), u(d, 0.0);
  for (int k = 0; k < d; ++k) hn[k] = f16_to_f64(h_new[k]);
  for (int r = 0; r < hd; ++r) {
    double acc = 0.0;
    for (int k = 0; k < d; ++k) acc += wq[(size_t)r * d + k] * hn[k];
    q[r] = acc;
  }
  for (int r = 0; r < hd; ++r)
    for (int k = 0; k < d; ++k) qt[k] += wk[(size_t)r * d + k] * q[r];
  const double inv = 1.0 / sqrt((double)hd);
  double m = -INFINITY;
  for (int64_t c = 0; c < n; ++c) {
    double dot = 0.0;
    for (int k = 0; k < d; ++k) dot += qt[k] * h_hat[c * d + k];
    s[c] = dot * inv;
    if (s[c] > m) m = s[c];
  }
  double Z = 0.0;
  for (int64_t c = 0; c < n; ++c) {
    s[c] = exp(s[c] - m);
    Z += s[c];
  }
  for (int64_t c = 0; c < n; ++c) {
    const double p = s[c] / Z;
    for (int k = 0; k < d; ++k) u[k] += p * h_hat[c * d + k];
  }
  for (int r = 0; r < hd; ++r) {
    double acc = 0.0;
    for (int k = 0; k < d; ++k) acc += wv[(size_t)r * d + k] * u[k];
    out_j[r] = acc;
  }
}

// Decode attention of one lane: h_hat [n][d] = the dequantised rows 0..n-1 of the iteration's
// layer (row n-1 is the new token, appended first), h_new fp16 [d]; out [H][hd].
// form 0 = explicit rebuild (the definition), 1 = absorbed.  Heads run on `threads` OpenMP
// threads (1 = single-threaded); each head is computed by one thread in the order above.
void oracle_attend(int form, int64_t n, int d, int H, int hd, const double* h_hat, const uint16_t* h_new,
                   const uint16_t* Wq, const uint16_t* Wk, const uint16_t* Wv, double* out, int threads) {
#pragma omp parallel for schedule(dynamic, 1) num_threads(threads > 0 ? threads : 1)
  for (int j = 0; j < H; ++j) {
    if (form == 0)
      attend_head_explicit(j, n, d, hd, h_hat, h_new, Wq, Wk, Wv, out + (size_t)j * hd);
    else
      attend_head_absorbed(j, n, d, hd, h_hat, h_new, Wq, Wk, Wv, out + (size_t)j * hd);
  }
}

// ---------------------------------------------------------------- safety check
// For each lane b with it < loops[b]: n2 = sum_k r_k^2 with every term exact in FP64; abort iff
// n2 > thr^2 (strict, thr taken as the fp32 value); flags sticky, first[b] = the first iteration
// that set the flag; norms[b] = sqrt(n2) (NaN for lanes left untouched).
void oracle_residual_norm_check(const float* residual, int B, int d, float threshold, int it, const int32_t* loops,
                                uint8_t* flags, int32_t* first, double* norms) {
  const double thr = (double)threshold;
  for (int b = 0; b < B; ++b) {
    norms[b] = NAN;
    if (it >= loops[b]) continue;
    double n2 = 0.0;
    for (int k = 0; k < d; ++k) {
      const double v = (double)residual[(size_t)b * d + k];
      n2 += v * v;
    }
    norms[b] = sqrt(n2);
    if (n2 > thr * thr) {
      if (flags[b] == 0) first[b] = it;
      flags[b] = 1;
    }
  }
}

// ---------------------------------------------------------------- one lane's decode iteration
// The whole path for one lane at one loop iteration, in the pages' order: the new token's h is
// quantised and appended at position n_ctx of the lane's rows of layer n_pre + it (codes /
// scales hold n_ctx + 1 rows; the first n_ctx are the cached context), all n_ctx + 1 rows are
// dequantised, attention runs over them (form as in oracle_attend), then the safety check.
// Returns the output in out [H][hd] and updates *flag / *first.
void oracle_decode_lane(int fmt, int d, int H, int hd, int64_t n_ctx, uint8_t* codes, void* scales,
                        const uint16_t* h_new, const uint16_t* Wq, const uint16_t* Wk, const uint16_t* Wv,
                        const float* residual, float threshold, int it, int loops, int form, double* out,
                        uint8_t* flag, int32_t* first, int threads) {
  const size_t cb = fmt == 0 ? 2 * (size_t)d : fmt == 1 ? (size_t)d : (size_t)d / 2;
  void* srow = fmt == 1 ? (void*)((float*)scales + n_ctx) : fmt == 2 ? (void*)((uint16_t*)scales + n_ctx * (d / 64))
                                                                     : nullptr;
  oracle_quantize_rows(fmt, d, 1, h_new, codes + n_ctx * cb, srow);
  std::vector<double> h_hat((size_t)(n_ctx + 1) * d);
  oracle_dequantize_rows(fmt, d, n_ctx + 1, codes, scales, h_hat.data());
  oracle_attend(form, n_ctx + 1, d, H, hd, h_hat.data(), h_new, Wq, Wk, Wv, out, threads);
  if (residual) {
    double norm;
    oracle_residual_norm_check(residual, 1, d, threshold, it, &loops, flag, first, &norm);
  }
}

// Exposed for the pins of the fp16 rounding above.
uint16_t oracle_f32_to_f16(float x) { return f32_to_f16_rne(x); }
double oracle_f16_to_f64(uint16_t h) { return f16_to_f64(h); }

int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

}  // extern "C"
