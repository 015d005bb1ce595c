/*
 * nvfp4_oracle.c -- plain CPU reference for the NVFP4 weight-only (W4A16)
 * linear layer and its round-to-nearest quantizer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: it exists so that tests, the smoke check and the CPU
 * baseline of the benchmark can compare the CUDA library against an
 * implementation that shares no code with it.  It is deliberately slow and
 * literal: values are decoded by table (E2M1) and by bit fields (E4M3),
 * rounding is done by searching the representable values, and dot products
 * are accumulated in fp64.
 *
 * Sources (web pages, by title and section):
 *   [p2] "Raphael Friedmann" home page, NVFP4 bit-level graphic: an E2M1
 *        element has one sign, two exponent and one mantissa bit (sixteen
 *        values); an FP8 scale per 16 values; an FP32 scale per tensor.
 *   [p3] imp docs/quantization.md: NVFP4 prequant = packed nibbles with FP8
 *        E4M3 micro-scales per 16 and an FP32 tensor scale (format table and
 *        the paragraph below it); imp-quantize writes .weight (U8 packed
 *        nibbles), .weight_scale (F8_E4M3), .weight_scale_2 (F32) and is plain
 *        round-to-nearest from the block absmax ("imp-quantize" section);
 *        the FP4 grid has eight magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6
 *        (micro-scale search paragraph); the decode GEMV reads packed FP4
 *        ("Dense layers" pipeline).
 *   [p5] model card "Qwen3.8-27B-NVFP4 (compressed-tensors)": weight-only
 *        NVFP4 with group size 16 and BF16 activations ("What is quantized");
 *        merged q/k/v and gate/up share one tensor scale (paragraph after the
 *        table).
 *
 * Readings where the pages leave a step open (each is also listed with the
 * design notes of the repository):
 *   R1  code -> value order of E2M1 follows the sign/exponent/mantissa fields
 *       of [p2]: bit 3 sign, bits 2..1 exponent (bias 1, subnormal at 0),
 *       bit 0 mantissa.
 *   R2  E4M3 is the finite-only FP8 variant: bias 7, subnormals m*2^-9,
 *       0x7F/0xFF are NaN, 0x7E = 448 is the largest value.  Scales are
 *       non-negative ("UE4M3" in [p3]).
 *   R3  packing: byte k/2 of a row holds element k in its low nibble and
 *       element k+1 in its high nibble; scale j covers elements 16j..16j+15;
 *       both arrays are row-major, unswizzled.
 *   R4  the tensor scale g is the dequantization multiplier amax / (6*448).
 *   R5  quantizer arithmetic is IEEE fp32, round to nearest even, in this
 *       order: s_f = (amax_b / 6) / g;  s = E4M3(s_f) saturating at 448;
 *       d = decode(s) * g;  r = 1 / d;  code = E2M1(w * r) saturating at 6,
 *       ties to the even code, sign kept.  g == 0 gives s = 0; d == 0 gives
 *       sixteen 0x0 codes; an input of +-0 gives code 0x0 / 0x8.
 *
 * MXFP4 ([p3] imp docs/quantization.md, the MXFP4 paragraph after the NVFP4
 * pipelines, and the MXFP4 row of the format table): the same E2M1 nibble
 * layout as NVFP4, one UE8M0 micro-scale per 32 elements, no tensor scale;
 * its quantizer is round-to-nearest.  The pages give no scale formula:
 *   R6  UE8M0 is an unsigned power of two: byte b means 2^(b - 127) for
 *       b = 0..254; 255 is NaN.
 *   R7  block scale X = 2^(floor(log2(amax_b)) - 2): 2 is the largest E2M1
 *       exponent (6 = 1.5 * 2^2), so the block's largest magnitude lands in
 *       [4, 8) before rounding.  The byte is clamped to 0..254; a block whose
 *       elements are all zero gets byte 0.
 *   R8  element codes: E2M1 round to nearest even of w / X (an exact
 *       division by a power of two, done in fp64), saturating at 6, sign kept
 *       (R5's rule).
 *   R9  packing as R3, with scale j covering elements 32j .. 32j+31.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- decode */

/* [p2]/[p3]: the sixteen E2M1 values, indexed by the 4-bit code (R1). */
static const double E2M1_VALUE[16] = {
    0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0,
    -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0,
};

double oracle_e2m1_decode(int code) { return E2M1_VALUE[code & 15]; }

/* [p2] FP8 scale, read as E4M3 by its bit fields (R2). */
double oracle_e4m3_decode(int byte) {
  int sign = (byte >> 7) & 1;
  int e = (byte >> 3) & 15;
  int m = byte & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    v = ldexp((double)m, -9);            /* subnormal: m/8 * 2^(1-7) */
  else
    v = ldexp(1.0 + m / 8.0, e - 7);     /* normal */
  return sign ? -v : v;
}

double oracle_bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

static float bf16_to_float(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* --------------------------------------------------------------- rounding */

/* Nearest of the non-negative E4M3 codes 0x00..0x7E to a (>= 0, finite,
 * <= 448), ties to the even code.  The codes are monotone in value, so a
 * binary search finds the largest code not above a, and the next one up is
 * the only other candidate. */
static int e4m3_nearest_code(double a) {
  int lo = 0, hi = 0x7E;
  while (lo < hi) {                     /* largest c with value(c) <= a */
    int mid = (lo + hi + 1) / 2;
    if (oracle_e4m3_decode(mid) <= a) lo = mid; else hi = mid - 1;
  }
  if (lo == 0x7E) return lo;
  double below = oracle_e4m3_decode(lo), above = oracle_e4m3_decode(lo + 1);
  double dl = a - below, du = above - a;
  if (dl < du) return lo;
  if (du < dl) return lo + 1;
  return (lo % 2 == 0) ? lo : lo + 1;   /* tie: even code */
}

/* E4M3 round-to-nearest-even with saturation to +-448 (R2, R5). */
int oracle_e4m3_rne_satfinite(float v) {
  int sign = signbit(v) ? 1 : 0;
  double a = fabs((double)v);
  int code;
  if (isnan(v)) return 0x7F;
  code = (a >= 448.0) ? 0x7E : e4m3_nearest_code(a);
  return (sign << 7) | code;
}

/* E2M1 round-to-nearest-even with saturation to +-6, sign kept (R5, R8). */
static int e2m1_rne_satfinite_d(double v) {
  int sign = signbit(v) ? 1 : 0;
  double a = fabs(v);
  int best = 0;
  if (a > 6.0) {
    best = 7;
  } else {
    for (int c = 1; c < 8; ++c) {       /* scan the eight magnitudes */
      double dc = fabs(E2M1_VALUE[c] - a), db = fabs(E2M1_VALUE[best] - a);
      if (dc < db || (dc == db && (c % 2 == 0))) best = c;
    }
  }
  return (sign << 3) | best;
}

int oracle_e2m1_rne_satfinite(float v) { return e2m1_rne_satfinite_d((double)v); }

/* ---------------------------------------------------------- tensor scale */

/* max |w| over rows x cols of a BF16 matrix with leading dimension ldw. */
float oracle_amax(const uint16_t* w, int64_t rows, int64_t cols, int64_t ldw) {
  float m = 0.0f;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c) {
      float a = fabsf(bf16_to_float(w[r * ldw + c]));
      if (a > m) m = a;
    }
  return m;
}

/* R4: g = amax / (6 * 448), one fp32 division. */
float oracle_tensor_scale(float amax) { return amax / 2688.0f; }

/* ------------------------------------------------------------- quantizer */

/* [p3] imp-quantize: round-to-nearest NVFP4 of a BF16 [N, K] matrix with
 * the tensor scale g given (for a merged layer, the members' shared g).
 * Writes q [N, K/2] and s [N, K/16].  K must be a multiple of 16. */
void oracle_quantize(const uint16_t* w, int64_t N, int64_t K, int64_t ldw,
                     float g, uint8_t* q, uint8_t* s) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t b = 0; b < K / 16; ++b) {
      const uint16_t* blk = w + n * ldw + b * 16;
      float amax_b = 0.0f;
      int codes[16];
      for (int i = 0; i < 16; ++i) {
        float a = fabsf(bf16_to_float(blk[i]));
        if (a > amax_b) amax_b = a;
      }
      int sc = 0;
      if (g != 0.0f) {
        float s_f = (amax_b / 6.0f) / g;
        sc = oracle_e4m3_rne_satfinite(s_f);
      }
      float d = (float)oracle_e4m3_decode(sc) * g;
      if (d == 0.0f) {
        for (int i = 0; i < 16; ++i) codes[i] = 0;
      } else {
        float r = 1.0f / d;
        for (int i = 0; i < 16; ++i) {
          float wi = bf16_to_float(blk[i]);
          if (wi == 0.0f)
            codes[i] = signbit(wi) ? 8 : 0;
          else
            codes[i] = oracle_e2m1_rne_satfinite(wi * r);
        }
      }
      s[n * (K / 16) + b] = (uint8_t)sc;
      for (int i = 0; i < 16; i += 2)
        q[n * (K / 2) + b * 8 + i / 2] = (uint8_t)(codes[i] | (codes[i + 1] << 4));
    }
  }
}

/* ------------------------------------------------ micro-scale search (MSE)
 *
 * [p3] micro-scale search paragraph: instead of taking the scale from the
 * block absmax, choose each micro-scale by minimising the block's
 * reconstruction error over FP8 candidates around the absmax scale (measured
 * there at about 6x the quantization cost for a 0.7% perplexity change, and
 * reverted).  The pages give no window, error precision or tie rule; the
 * readings taken:
 *   - candidates: the E4M3 codes c with |c - c0| <= window, clamped to
 *     1..126, where c0 is the round-to-nearest code of oracle_quantize
 *     (window 8 = one binade of E4M3 either side of it);
 *   - each candidate quantizes the block as the round-to-nearest rule does
 *     with its scale: d = e4m3(c) * g in fp32, r = 1 / d, codes = E2M1 RNE of
 *     w * r (zeros keep their sign);
 *   - its error is sum_i (w_i - e2m1(code_i) * d)^2 in fp64, summed in index
 *     order with no contraction;
 *   - the smallest error wins; ties go to the code nearest c0, then to the
 *     smaller code;
 *   - a block whose c0 is 0 (zero block, or g = 0) stays as the
 *     round-to-nearest rule leaves it (scale 0, codes 0).
 * window = 0 reproduces oracle_quantize exactly. */
static void rtn_codes(const float* f, float d, int* codes) {
  const float r = 1.0f / d;
  for (int i = 0; i < 16; ++i) {
    if (f[i] == 0.0f)
      codes[i] = signbit(f[i]) ? 8 : 0;
    else
      codes[i] = oracle_e2m1_rne_satfinite(f[i] * r);
  }
}

void oracle_quantize_mse(const uint16_t* w, int64_t N, int64_t K, int64_t ldw, float g, int window,
                         uint8_t* q, uint8_t* s) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t b = 0; b < K / 16; ++b) {
      const uint16_t* blk = w + n * ldw + b * 16;
      float f[16];
      float amax_b = 0.0f;
      for (int i = 0; i < 16; ++i) {
        f[i] = bf16_to_float(blk[i]);
        if (fabsf(f[i]) > amax_b) amax_b = fabsf(f[i]);
      }
      int c0 = 0;
      if (g != 0.0f) c0 = oracle_e4m3_rne_satfinite((amax_b / 6.0f) / g);
      int best_c = 0, best_codes[16];
      for (int i = 0; i < 16; ++i) best_codes[i] = 0;
      if (c0 != 0) {
        double best_err = INFINITY;
        const int lo = c0 - window < 1 ? 1 : c0 - window;
        const int hi = c0 + window > 126 ? 126 : c0 + window;
        for (int c = lo; c <= hi; ++c) {
          const float d = (float)oracle_e4m3_decode(c) * g;
          if (d == 0.0f) continue;
          int codes[16];
          rtn_codes(f, d, codes);
          double err = 0.0;
          for (int i = 0; i < 16; ++i) {
            const double e = (double)f[i] - E2M1_VALUE[codes[i]] * (double)d;
            err += e * e;
          }
          const int dc = abs(c - c0), db = abs(best_c - c0);
          if (err < best_err || (err == best_err && (dc < db || (dc == db && c < best_c)))) {
            best_err = err;
            best_c = c;
            for (int i = 0; i < 16; ++i) best_codes[i] = codes[i];
          }
        }
      }
      s[n * (K / 16) + b] = (uint8_t)best_c;
      for (int i = 0; i < 16; i += 2)
        q[n * (K / 2) + b * 8 + i / 2] = (uint8_t)(best_codes[i] | (best_codes[i + 1] << 4));
    }
  }
}

/* ---------------------------------------------------- dequant and product */

/* W_deq[n, k] = g * e4m3(s[n, k/16]) * e2m1(q[n, k]) in fp64. */
void oracle_dequantize(const uint8_t* q, const uint8_t* s, float g, int64_t N,
                       int64_t K, double* out) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) {
      uint8_t byte = q[n * (K / 2) + k / 2];
      int code = (k % 2 == 0) ? (byte & 15) : (byte >> 4);
      out[n * K + k] = (double)g * oracle_e4m3_decode(s[n * (K / 16) + k / 16]) *
                       oracle_e2m1_decode(code);
    }
}

/* [p5] W4A16 linear, y = x . W^T, for the output elements listed in
 * (rows m_idx[i], columns n_idx[i]); all of them when count < 0 (then the
 * result is [M, N] row-major).  For each output:
 *   y[m, n]   = g * sum_b e4m3(s[n, b]) * sum_i e2m1(q[n, 16b+i]) * x[m, 16b+i]
 *   bound[m,n] = sum_k |W_deq[n, k] * x[m, k]|
 * both in fp64 (every product is exact in fp64). */
void oracle_linear(const uint16_t* x, int64_t ldx, const uint8_t* q,
                   const uint8_t* s, float g, int64_t M, int64_t N, int64_t K,
                   const int64_t* m_idx, const int64_t* n_idx, int64_t count,
                   double* y, double* bound) {
  int64_t total = count < 0 ? M * N : count;
#pragma omp parallel for schedule(dynamic, 64)
  for (int64_t t = 0; t < total; ++t) {
    int64_t m = count < 0 ? t / N : m_idx[t];
    int64_t n = count < 0 ? t % N : n_idx[t];
    double acc = 0.0, mag = 0.0;
    for (int64_t b = 0; b < K / 16; ++b) {
      double sb = oracle_e4m3_decode(s[n * (K / 16) + b]);
      double part = 0.0, part_mag = 0.0;
      for (int i = 0; i < 16; ++i) {
        int64_t k = b * 16 + i;
        uint8_t byte = q[n * (K / 2) + k / 2];
        int code = (k % 2 == 0) ? (byte & 15) : (byte >> 4);
        double prod = oracle_e2m1_decode(code) * oracle_bf16_to_double(x[m * ldx + k]);
        part += prod;
        part_mag += fabs(prod);
      }
      acc += sb * part;
      mag += sb * part_mag;
    }
    y[t] = (double)g * acc;
    bound[t] = fabs((double)g) * mag;
  }
}

/* ------------------------------------------------------------------ MXFP4 */

/* R6: UE8M0 byte -> 2^(b - 127); 255 is NaN. */
double oracle_e8m0_decode(int byte) {
  byte &= 255;
  return byte == 255 ? NAN : ldexp(1.0, byte - 127);
}

/* [p3] round-to-nearest MXFP4 of a BF16 [N, K] matrix (K a multiple of 32):
 * q [N, K/2] as R3, s [N, K/32] UE8M0 bytes (R7), codes by R8. */
void oracle_mx_quantize(const uint16_t* w, int64_t N, int64_t K, int64_t ldw,
                        uint8_t* q, uint8_t* s) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t b = 0; b < K / 32; ++b) {
      const uint16_t* blk = w + n * ldw + b * 32;
      double amax_b = 0.0;
      int codes[32];
      for (int i = 0; i < 32; ++i) {
        double a = fabs(oracle_bf16_to_double(blk[i]));
        if (a > amax_b) amax_b = a;
      }
      int byte = 0;
      if (amax_b > 0.0) {
        int e2;                       /* amax_b = m * 2^e2 with m in [0.5, 1) */
        frexp(amax_b, &e2);
        int e = (e2 - 1) - 2;         /* floor(log2(amax_b)) - 2 */
        byte = e + 127;
        if (byte < 0) byte = 0;
        if (byte > 254) byte = 254;
      }
      double x_scale = oracle_e8m0_decode(byte);
      for (int i = 0; i < 32; ++i) {
        double wi = oracle_bf16_to_double(blk[i]);
        codes[i] = e2m1_rne_satfinite_d(wi / x_scale);
      }
      s[n * (K / 32) + b] = (uint8_t)byte;
      for (int i = 0; i < 32; i += 2)
        q[n * (K / 2) + b * 16 + i / 2] = (uint8_t)(codes[i] | (codes[i + 1] << 4));
    }
  }
}

/* W_deq[n, k] = e8m0(s[n, k/32]) * e2m1(q[n, k]) in fp64. */
void oracle_mx_dequantize(const uint8_t* q, const uint8_t* s, int64_t N, int64_t K, double* out) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) {
      uint8_t byte = q[n * (K / 2) + k / 2];
      int code = (k % 2 == 0) ? (byte & 15) : (byte >> 4);
      out[n * K + k] = oracle_e8m0_decode(s[n * (K / 32) + k / 32]) * oracle_e2m1_decode(code);
    }
}

/* MXFP4 weight-only linear, y = x . W^T, outputs selected as in
 * oracle_linear:
 *   y[m, n]    = sum_b e8m0(s[n, b]) * sum_i e2m1(q[n, 32b+i]) * x[m, 32b+i]
 *   bound[m,n] = sum_k |W_deq[n, k] * x[m, k]|      (fp64) */
void oracle_mx_linear(const uint16_t* x, int64_t ldx, const uint8_t* q, const uint8_t* s,
                      int64_t M, int64_t N, int64_t K, const int64_t* m_idx, const int64_t* n_idx,
                      int64_t count, double* y, double* bound) {
  int64_t total = count < 0 ? M * N : count;
#pragma omp parallel for schedule(dynamic, 64)
  for (int64_t t = 0; t < total; ++t) {
    int64_t m = count < 0 ? t / N : m_idx[t];
    int64_t n = count < 0 ? t % N : n_idx[t];
    double acc = 0.0, mag = 0.0;
    for (int64_t b = 0; b < K / 32; ++b) {
      double sb = oracle_e8m0_decode(s[n * (K / 32) + b]);
      double part = 0.0, part_mag = 0.0;
      for (int i = 0; i < 32; ++i) {
        int64_t k = b * 32 + i;
        uint8_t byte = q[n * (K / 2) + k / 2];
        int code = (k % 2 == 0) ? (byte & 15) : (byte >> 4);
        double prod = oracle_e2m1_decode(code) * oracle_bf16_to_double(x[m * ldx + k]);
        part += prod;
        part_mag += fabs(prod);
      }
      acc += sb * part;
      mag += sb * part_mag;
    }
    y[t] = acc;
    bound[t] = mag;
  }
}

/* Threads the OpenMP loops above run on (1 without OpenMP). */
int oracle_num_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}
