/*
 * fh_oracle.c -- plain CPU oracle for the NVFP4 quantized linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or constant with the CUDA library, and it never reads
 * anything the CUDA library produced except through the parity tests'
 * explicit comparisons.
 *
 * What it computes, and where that comes from:
 *
 *  - FastH3 thread digest (farwalk.ai), tweet 5/8: on Blackwell the
 *    transformer's linear layers run in NVFP4.
 *  - FastH3 thread digest (farwalk.ai), tweet 6/8: with uncalibrated FP4
 *    scales the activations clip (40 of 42 blocks, worst 137x the limit);
 *    calibrating every FP4 layer on 1,000 prompts keeps them intact.
 *  - FastH3 Trim (comfyui-wiki news), "What the ComfyUI repack contains":
 *    every NVFP4 layer carries an activation scale calibrated on 1,000
 *    prompts (294 calibrated layers in Trim).
 *
 * The pages name NVFP4 but never define it.  The definition used here is the
 * public one: 4-bit E2M1 elements (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6),
 * one unsigned E4M3 scale (FN variant, max 448) per 16 consecutive elements
 * along K, and one FP32 global scale per tensor.  Every rounding decision is
 * taken on the EXACT real quotient (round to nearest, ties to the even code),
 * evaluated by exact comparisons in binary64: each threshold below is a
 * product of numbers with at most 31 significant bits in total, so binary64
 * holds it exactly and the comparison with a BF16 input is exact.
 *
 * Everything is a plain loop in the order the definition states; the GEMM is
 * the dequantized product summed in binary64 (no blocking, no reordering).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define FP4_MAX 6.0
#define E4M3_MAX 448.0
#define E4M3_MAX_CODE 0x7E

/* ---------------------------------------------------------------------- */
/* Element formats                                                        */
/* ---------------------------------------------------------------------- */

/* BF16 bit pattern -> its exact value (BF16 is the top half of an FP32). */
double oracle_bf16_value(uint16_t bits) {
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* E2M1 code (bit 3 sign, bits 2..1 exponent with bias 1, bit 0 mantissa).
 * Exponent 0 is subnormal: 0.5 * mantissa.  No Inf, no NaN. */
double oracle_e2m1_value(int code) {
  int mag = code & 7;
  int e = (mag >> 1) & 3;
  int m = mag & 1;
  double v = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
  return (code & 8) ? -v : v;
}

/* E4M3 "FN" byte: bit 7 sign, bits 6..3 exponent with bias 7, bits 2..0
 * mantissa.  Exponent 0 is subnormal (m * 2^-9).  0x7F / 0xFF are NaN; there
 * is no Inf, so the largest finite magnitude is 1.75 * 2^8 = 448. */
double oracle_e4m3_value(int byte) {
  int s = (byte >> 7) & 1;
  int e = (byte >> 3) & 15;
  int m = byte & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    v = ldexp((double)m, -9);
  else
    v = ldexp(1.0 + m / 8.0, e - 7);
  return s ? -v : v;
}

/* Round q >= 0 to the nearest non-negative E4M3 value, ties to the even
 * code (mantissa bit 0), saturating: q >= 448 gives 448.  The code c wins over
 * c-1 when q lies above their midpoint, or on it with c even. */
int oracle_e4m3_rne_sat(double q) {
  int best = 0;
  for (int c = 1; c <= E4M3_MAX_CODE; ++c) {
    double mid = 0.5 * (oracle_e4m3_value(c - 1) + oracle_e4m3_value(c));
    if (q > mid || (q == mid && (c % 2) == 0)) best = c;
  }
  return best;
}

/* Round r >= 0 to the nearest E2M1 magnitude code (0..7), ties to the even
 * code, saturating at 6. */
int oracle_e2m1_rne_sat(double r) {
  int best = 0;
  for (int c = 1; c <= 7; ++c) {
    double mid = 0.5 * (oracle_e2m1_value(c - 1) + oracle_e2m1_value(c));
    if (r > mid || (r == mid && (c % 2) == 0)) best = c;
  }
  return best;
}

/* ---------------------------------------------------------------------- */
/* Calibration: global scale from a calibrated amax                        */
/* ---------------------------------------------------------------------- */

/* The global scale maps the calibrated amax onto the largest representable
 * magnitude 6 * 448 = 2688 (FastH3 thread digest, tweet 6/8: calibrated scales
 * keep large activations intact).  Reading: s_g is the SMALLEST FP32 value with
 * 2688 * s_g >= amax, so an element no larger than the calibrated amax is never
 * clipped.  amax == 0 gives s_g = 1.  amax must be finite. */
float oracle_scale_from_amax(float amax) {
  if (!(amax > 0.0f)) return 1.0f;
  const double A = (double)amax;
  float s = (float)(A / (FP4_MAX * E4M3_MAX));
  while ((double)s * (FP4_MAX * E4M3_MAX) < A) s = nextafterf(s, INFINITY);
  while (s > 0.0f && (double)nextafterf(s, 0.0f) * (FP4_MAX * E4M3_MAX) >= A)
    s = nextafterf(s, 0.0f);
  return s;
}

/* max |x| over a row-major BF16 matrix (rows x cols, leading dimension ld). */
float oracle_amax(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld) {
  double amax = 0.0;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c) {
      double a = fabs(oracle_bf16_value(x[r * ld + c]));
      if (a > amax) amax = a;
    }
  return (float)amax; /* exact: amax is a BF16 value */
}

/* ---------------------------------------------------------------------- */
/* Quantization of one row-major BF16 matrix                              */
/* ---------------------------------------------------------------------- */

/* Block scale: S_b = E4M3 RNE (saturating) of amax_b / (6 * s_g).
 * Compared as amax_b against mid * 6 * s_g, which is exact in binary64; the
 * boundaries t[c] = mid(c-1, c) * 6 * s_g depend on s_g only, so a call
 * computes them once (scale_boundaries) and every block compares with them. */
static void scale_boundaries(double sg, double t[E4M3_MAX_CODE + 1]) {
  t[0] = 0.0;
  for (int c = 1; c <= E4M3_MAX_CODE; ++c) {
    double mid = 0.5 * (oracle_e4m3_value(c - 1) + oracle_e4m3_value(c));
    t[c] = mid * FP4_MAX * sg;
  }
}

static int block_scale_code(double amax_b, const double t[E4M3_MAX_CODE + 1]) {
  int best = 0;
  for (int c = 1; c <= E4M3_MAX_CODE; ++c)
    if (amax_b > t[c] || (amax_b == t[c] && (c % 2) == 0)) best = c;
  return best;
}

/* Element code: sign bit = sign bit of x (so -0 and small negatives give 8);
 * magnitude = E2M1 RNE (saturating at 6) of |x| / (S_b * s_g), compared as
 * |x| against mid * S_b * s_g (exact in binary64).  S_b == 0 gives magnitude
 * 0.  The seven boundaries t[c] = mid(c-1, c) * S_b * s_g are the block's, so
 * a block computes them once (element_boundaries). */
static void element_boundaries(double S, double sg, double t[8]) {
  t[0] = 0.0;
  for (int c = 1; c <= 7; ++c) {
    double mid = 0.5 * (oracle_e2m1_value(c - 1) + oracle_e2m1_value(c));
    t[c] = mid * S * sg;
  }
}

static int element_code(double x, double S, const double t[8]) {
  int sign = signbit(x) ? 8 : 0;
  double a = fabs(x);
  if (S == 0.0) return sign;
  int best = 0;
  for (int c = 1; c <= 7; ++c)
    if (a > t[c] || (a == t[c] && (c % 2) == 0)) best = c;
  return sign | best;
}

/* Quantize x [M, K] (leading dimension ldx, K a multiple of 16) with global
 * scale sg.  Outputs:
 *   codes  [M, K/2] bytes, element 2j in the low nibble, 2j+1 in the high one;
 *   scales [M, K/16] E4M3 bytes, row-major;
 *   *clip  += number of elements with |x| > 2688 * sg (beyond the largest
 *             magnitude the scaled format can represent). */
void oracle_quantize(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                     float sg_f, uint8_t* codes, uint8_t* scales,
                     uint64_t* clip) {
  const double sg = (double)sg_f;
  const double limit = FP4_MAX * E4M3_MAX * sg; /* exact */
  const int64_t nb = K / 16;
  uint64_t nclip = 0;
  double st[E4M3_MAX_CODE + 1];
  scale_boundaries(sg, st);
  /* Rows are independent; the clip count is an integer sum. */
#pragma omp parallel for schedule(static) reduction(+ : nclip)
  for (int64_t m = 0; m < M; ++m) {
    const uint16_t* row = x + m * ldx;
    for (int64_t b = 0; b < nb; ++b) {
      double amax = 0.0;
      for (int i = 0; i < 16; ++i) {
        double a = fabs(oracle_bf16_value(row[16 * b + i]));
        if (a > amax) amax = a;
      }
      int sc = block_scale_code(amax, st);
      double S = oracle_e4m3_value(sc);
      double et[8];
      element_boundaries(S, sg, et);
      scales[m * nb + b] = (uint8_t)sc;
      for (int i = 0; i < 16; i += 2) {
        double x0 = oracle_bf16_value(row[16 * b + i]);
        double x1 = oracle_bf16_value(row[16 * b + i + 1]);
        int c0 = element_code(x0, S, et);
        int c1 = element_code(x1, S, et);
        codes[m * (K / 2) + 8 * b + i / 2] = (uint8_t)(c0 | (c1 << 4));
        if (fabs(x0) > limit) ++nclip;
        if (fabs(x1) > limit) ++nclip;
      }
    }
  }
  *clip += nclip;
}

/* Clip count alone: the number of elements of x [M, K] (leading dimension
 * ldx) with |x| > 2688 * sg, the largest magnitude the scaled format can
 * represent (the same count oracle_quantize adds to *clip). */
uint64_t oracle_clip_count(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, float sg_f) {
  const double limit = FP4_MAX * E4M3_MAX * (double)sg_f; /* exact */
  uint64_t n = 0;
#pragma omp parallel for schedule(static) reduction(+ : n)
  for (int64_t m = 0; m < M; ++m)
    for (int64_t k = 0; k < K; ++k)
      if (fabs(oracle_bf16_value(x[m * ldx + k])) > limit) ++n;
  return n;
}

/* Dequantize a quantized [rows, K] matrix row r into out[0..K): the E2M1 value
 * of each code times its block's E4M3 scale (exact in binary64). */
static void dequant_row(const uint8_t* codes, const uint8_t* scales, int64_t K,
                        int64_t r, double* out) {
  for (int64_t k = 0; k < K; ++k) {
    uint8_t byte = codes[r * (K / 2) + k / 2];
    int code = (k % 2 == 0) ? (byte & 15) : (byte >> 4);
    out[k] = oracle_e2m1_value(code) * oracle_e4m3_value(scales[r * (K / 16) + k / 16]);
  }
}

/* ---------------------------------------------------------------------- */
/* Linear layer: y = s_gA * s_gW * (A_deq . W_deq^T) + bias, in binary64  */
/* ---------------------------------------------------------------------- */

/* For each requested row index rows[i] (0 <= rows[i] < M) and every n < N:
 *   y  [i, n] = a_g * w_g * sum_k A[rows[i], k] * W[n, k] + bias[n]
 *   mag[i, n] = |a_g * w_g| * sum_k |A[rows[i], k] * W[n, k]|
 * where A and W are the dequantized operands (E2M1 value times the block's
 * E4M3 scale) and bias may be NULL (zero).  Scales are row-major.
 * w_deq is caller-provided scratch of N*K doubles, a_deq of nrows*K doubles. */
void oracle_linear(const uint8_t* a_codes, const uint8_t* a_scales, float a_g,
                   const uint8_t* w_codes, const uint8_t* w_scales, float w_g,
                   const uint16_t* bias, int64_t N, int64_t K,
                   const int64_t* rows, int64_t nrows, double* w_deq,
                   double* a_deq, double* y, double* mag) {
  const double alpha = (double)a_g * (double)w_g;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) dequant_row(w_codes, w_scales, K, n, w_deq + n * K);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < nrows; ++i) dequant_row(a_codes, a_scales, K, rows[i], a_deq + i * K);
#pragma omp parallel for collapse(2) schedule(static)
  for (int64_t i = 0; i < nrows; ++i) {
    for (int64_t n = 0; n < N; ++n) {
      const double* a = a_deq + i * K;
      const double* w = w_deq + n * K;
      double acc = 0.0, acc_abs = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        double p = a[k] * w[k];
        acc += p;
        acc_abs += fabs(p);
      }
      double b = bias ? oracle_bf16_value(bias[n]) : 0.0;
      y[i * N + n] = alpha * acc + b;
      mag[i * N + n] = fabs(alpha) * acc_abs;
    }
  }
}

/* Exact-erf GELU in binary64: y = x * Phi(x) = x/2 * (1 + erf(x / sqrt 2)),
 * evaluated as x/2 * erfc(-x / sqrt 2), the same function written so that the
 * negative tail (where 1 + erf cancels to 0) keeps its value. */
void oracle_gelu(const uint16_t* x, int64_t n, double* y) {
  for (int64_t i = 0; i < n; ++i) {
    double v = oracle_bf16_value(x[i]);
    y[i] = 0.5 * v * erfc(-v / sqrt(2.0));
  }
}
