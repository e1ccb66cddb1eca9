// fh_nvfp4.cuh -- the NVFP4 block quantization shared by the stand-alone
// quantizer (fh_quant.cu) and the GEMM epilogue that emits the next layer's
// NVFP4 input (fh_gemm.cu), so both produce the same codes, scales and clip
// counts from the same BF16 values.
//
// Rules (FastH3 thread digest, farwalk.ai, tweet 6/8, and FastH3 Trim,
// comfyui-wiki news, "What the ComfyUI repack contains": every FP4 layer's
// input is quantized with a calibrated per-layer scale s_g): per 16-element
// block, S_b = E4M3(amax_b / (6 s_g)) and code = E2M1(x / (S_b s_g)), both to
// nearest with ties to the even code on the EXACT quotient, saturating at 448
// and 6; the code's sign bit is the sign bit of x; |x| > 2688 s_g is clipped.
//
// Every rounding decision compares a BF16 magnitude with an exact threshold;
// the host builds those thresholds (QuantTable) in FP64 for each s_g.  Blocks
// go through the hardware converter on x * (1/(S s_g)) for scale codes where
// the host proved the converter exact at every decision boundary, and through
// integer threshold compares otherwise.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace fh {

struct __align__(16) QuantTable {
  uint16_t code_thr[128][8];  // [c][j<7]: smallest |x| (BF16 bits) whose exact magnitude code is >= j+1 at scale code c
  // Per scale code c, everything one block needs in one 8-byte load:
  //   x: the FP32 bits of 1 / (S_c * s_g), the multiplier of the converter path
  //      (0 for c == 0);
  //   y: bits 0..14 the smallest block amax (BF16 magnitude bits) whose exact
  //      scale code is >= c, bit 15 set when the converter path is exact at c,
  //      bits 16..30 the same threshold for code c + 1 (+Inf bits for c = 126).
  uint2 sc[128];
};
static_assert(sizeof(QuantTable) % 16 == 0, "table copy granularity");

namespace nvfp4 {

// E4M3 x2 conversion (round to nearest even, saturating); the low byte's code.
__device__ __forceinline__ uint32_t cvt_e4m3_sat(float v) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
  return r & 0xFFu;
}

// max(|a|, |b|) per BF16 half (sign bits = xor of the inputs' signs).
__device__ __forceinline__ uint32_t max_abs_bf16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ float bf16_to_float(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

// 16 BF16 values (words w0..w7 in q0, q1) -> 8 code bytes, exact-threshold path.
// Out of line: only blocks whose scale code failed the converter check get here.
static __device__ __noinline__ uint2 codes_exact(const QuantTable& t, uint32_t c, uint4 q0, uint4 q1) {
  const uint32_t w[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
  uint32_t thr[7];
#pragma unroll
  for (int j = 0; j < 7; ++j) thr[j] = t.code_thr[c][j];
  uint32_t out[2] = {0, 0};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t lo = w[i] & 0xFFFFu, hi = w[i] >> 16;
    uint32_t ml = 0, mh = 0;
#pragma unroll
    for (int j = 0; j < 7; ++j) {
      ml += ((lo & 0x7FFFu) >= thr[j]) ? 1u : 0u;
      mh += ((hi & 0x7FFFu) >= thr[j]) ? 1u : 0u;
    }
    const uint32_t byte = (ml | ((lo >> 12) & 8u)) | ((mh | ((hi >> 12) & 8u)) << 4);
    out[i >> 2] |= byte << (8 * (i & 3));
  }
  return make_uint2(out[0], out[1]);
}

// Four BF16 words (8 values) -> 4 code bytes (low value in the low nibble);
// the products x * inv are formed two at a time (mul.rn.f32x2: IEEE
// round-to-nearest per lane, no flush to zero, the same as a scalar multiply).
__device__ __forceinline__ uint32_t cvt_e2m1x8(float inv, uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3) {
  uint32_t r;
  asm("{\n\t.reg .b64 s, a0, a1, a2, a3;\n\t.reg .f32 l0, h0, l1, h1, l2, h2, l3, h3;\n\t.reg .b8 t0, t1, t2, t3;\n\t"
      "mov.b64 s, {%9, %9};\n\t"
      "mov.b64 a0, {%1, %2};\n\tmov.b64 a1, {%3, %4};\n\tmov.b64 a2, {%5, %6};\n\tmov.b64 a3, {%7, %8};\n\t"
      "mul.rn.f32x2 a0, a0, s;\n\tmul.rn.f32x2 a1, a1, s;\n\tmul.rn.f32x2 a2, a2, s;\n\tmul.rn.f32x2 a3, a3, s;\n\t"
      "mov.b64 {l0, h0}, a0;\n\tmov.b64 {l1, h1}, a1;\n\tmov.b64 {l2, h2}, a2;\n\tmov.b64 {l3, h3}, a3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t0, h0, l0;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t1, h1, l1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t2, h2, l2;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t3, h3, l3;\n\t"
      "mov.b32 %0, {t0, t1, t2, t3};\n\t}"
      : "=r"(r)
      : "f"(__uint_as_float(w0 << 16)), "f"(__uint_as_float(w0 & 0xFFFF0000u)),
        "f"(__uint_as_float(w1 << 16)), "f"(__uint_as_float(w1 & 0xFFFF0000u)),
        "f"(__uint_as_float(w2 << 16)), "f"(__uint_as_float(w2 & 0xFFFF0000u)),
        "f"(__uint_as_float(w3 << 16)), "f"(__uint_as_float(w3 & 0xFFFF0000u)), "f"(inv));
  return r;
}

// One 16-element block, BF16 words w[0..7] (element 2i in the low half of
// w[i]): returns the scale code and sets the 8 code bytes (element 2j in the
// low nibble of byte j).  inv6sg = 1 / (6 s_g) gives the scale-code candidate.
__device__ __forceinline__ uint32_t quantize_block_codes(const QuantTable& tab, float inv6sg, const uint32_t* w,
                                                         uint32_t& amax_bits, uint2& codes) {
  // Block amax over the magnitudes (a max, so exact).
  const uint32_t r01 = max_abs_bf16x2(w[0], w[1]), r23 = max_abs_bf16x2(w[2], w[3]);
  const uint32_t r45 = max_abs_bf16x2(w[4], w[5]), r67 = max_abs_bf16x2(w[6], w[7]);
  const uint32_t r = max_abs_bf16x2(max_abs_bf16x2(r01, r23), max_abs_bf16x2(r45, r67));
  const uint32_t amax = max_abs_bf16x2(r, __byte_perm(r, 0, 0x1032)) & 0x7FFFu;
  // Scale code: converter candidate, corrected against the exact thresholds
  // (the candidate is almost always right: one table load checks it).
  const float amax_f = bf16_to_float(amax);
  uint32_t c = min(cvt_e4m3_sat(amax_f * inv6sg), 126u);
  uint2 e = tab.sc[c];
  if (amax < (e.y & 0x7FFFu) || amax >= (e.y >> 16)) {
    while (c < 126u && amax >= (tab.sc[c].y >> 16)) ++c;
    while (c > 0u && amax < (tab.sc[c].y & 0x7FFFu)) --c;
    e = tab.sc[c];
  }
  const float inv = __uint_as_float(e.x);
  if (((e.y >> 15) & 1u) && (amax_f * inv <= 3.0e38f)) {
    codes = make_uint2(cvt_e2m1x8(inv, w[0], w[1], w[2], w[3]), cvt_e2m1x8(inv, w[4], w[5], w[6], w[7]));
  } else {
    codes = codes_exact(tab, c, make_uint4(w[0], w[1], w[2], w[3]), make_uint4(w[4], w[5], w[6], w[7]));
  }
  amax_bits = amax;
  return c;
}

// Elements of the block with |x| > 2688 s_g (clip_thr: the smallest such BF16
// magnitude); only blocks whose amax reaches it can hold any.
__device__ __forceinline__ uint32_t block_clips(const uint32_t* w, uint32_t amax_bits, uint32_t clip_thr) {
  uint32_t n = 0;
  if (amax_bits >= clip_thr) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      n += ((w[i] & 0x7FFFu) >= clip_thr) ? 1u : 0u;
      n += (((w[i] >> 16) & 0x7FFFu) >= clip_thr) ? 1u : 0u;
    }
  }
  return n;
}

// GELU of both BF16 halves of w (the low half is the first element), rounded
// to BF16 and packed the same way:
//   GELU(x) = x/2 * erfc(-x/sqrt 2) = x/2 * (1 + erf(x/sqrt 2)),
// using erfc(-x/sqrt 2) = 2 - erfc(x/sqrt 2) for x >= 0, so there is no
// 1 + erf cancellation for negative x.  erfc(z), z >= 0, takes the
// Chebyshev-fitted form
//   erfc(z) ~= t * exp(-z^2 + P(t)),  t = 1 / (1 + z/2),
// with P of degree 9, whose fractional error is below 1.2e-7 for every z >= 0
// (Press, Teukolsky, Vetterling and Flannery, Numerical Recipes, 2nd ed.,
// section 6.2).  In FP32 with the hardware reciprocal and base-2 exponent the
// relative error stays near 1e-6, far below BF16's 2^-8; values below the FP32
// normal range flush to zero.  The two elements go through the packed FP32x2
// pipe together.
__device__ __forceinline__ float ex2_approx(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ uint32_t gelu2_bits(uint32_t w) {
  const float2 v = make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
  const float2 z = __fmul2_rn(make_float2(__uint_as_float((w << 16) & 0x7FFFFFFFu),
                                          __uint_as_float(w & 0x7FFF0000u)),
                              make_float2(0.70710678118654752440f, 0.70710678118654752440f));
  const float2 d = __ffma2_rn(make_float2(0.5f, 0.5f), z, make_float2(1.0f, 1.0f));
  const float2 t = make_float2(__fdividef(1.0f, d.x), __fdividef(1.0f, d.y));
  float2 p = make_float2(0.17087277f, 0.17087277f);
  p = __ffma2_rn(p, t, make_float2(-0.82215223f, -0.82215223f));
  p = __ffma2_rn(p, t, make_float2(1.48851587f, 1.48851587f));
  p = __ffma2_rn(p, t, make_float2(-1.13520398f, -1.13520398f));
  p = __ffma2_rn(p, t, make_float2(0.27886807f, 0.27886807f));
  p = __ffma2_rn(p, t, make_float2(-0.18628806f, -0.18628806f));
  p = __ffma2_rn(p, t, make_float2(0.09678418f, 0.09678418f));
  p = __ffma2_rn(p, t, make_float2(0.37409196f, 0.37409196f));
  p = __ffma2_rn(p, t, make_float2(1.00002368f, 1.00002368f));
  p = __ffma2_rn(p, t, make_float2(-1.26551223f, -1.26551223f));
  // exp(-z^2 + P) = 2^((-z^2 + P) * log2(e))
  const float2 a = __fmul2_rn(__ffma2_rn(make_float2(-z.x, -z.y), z, p),
                              make_float2(1.44269504088896340736f, 1.44269504088896340736f));
  const float2 e = __fmul2_rn(t, make_float2(ex2_approx(a.x), ex2_approx(a.y)));
  const float2 phi2 = make_float2(v.x >= 0.0f ? 2.0f - e.x : e.x, v.y >= 0.0f ? 2.0f - e.y : e.y);
  const float2 y = __fmul2_rn(__fmul2_rn(make_float2(0.5f, 0.5f), v), phi2);
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(y.y), "f"(y.x));
  return r;
}

// GELU of one BF16 value (low 16 bits), rounded to BF16: the same arithmetic
// as gelu2_bits.
__device__ __forceinline__ uint32_t gelu_bits(uint32_t bits16) { return gelu2_bits(bits16 & 0xFFFFu) & 0xFFFFu; }

}  // namespace nvfp4
}  // namespace fh
