// fh_quant.cu -- NVFP4 activation quantizer, calibration amax, scale relayout
// and the BF16 GELU used between the two FFN linear layers.
//
// Quantizer (FastH3 thread digest, farwalk.ai, tweet 6/8, and FastH3 Trim,
// comfyui-wiki news, "What the ComfyUI repack contains": every FP4 layer's
// activations are quantized with a calibrated per-layer scale).  Per 16-element
// block along K: S_b = E4M3(amax_b / (6 s_g)) and code = E2M1(x / (S_b s_g)),
// both to nearest with ties to the even code on the EXACT quotient, saturating
// at 448 and 6; the code's sign bit is the sign bit of x.  Elements with
// |x| > 2688 s_g are counted as clipped.
//
// How the exact rounding stays cheap.  The inputs are BF16, so every decision
// "is |x| (or amax_b) on this side of the exact real threshold t * S * s_g" is
// the same as an integer compare of |x|'s 15 magnitude bits with the smallest
// BF16 at (or beyond) the threshold.  Each CTA first builds, from s_g in FP64
// (where t * S * s_g is exact), these BF16 decision thresholds for all 126
// finite non-zero scale codes.  For the elements it then uses the hardware
// converter on x * (1 / (S s_g)) -- one multiply per element, two elements per
// cvt -- but only for scale codes where it has checked, at every decision
// boundary, that the converter's answer equals the exact one; the converter
// and the multiply are monotone, so agreement at both sides of every boundary
// means agreement on every BF16 input.  Blocks whose scale code failed the
// check (exact ties at non-power-of-two scales, typically) take the exact
// threshold-compare path instead.  The block scale itself takes a converter
// candidate and corrects it against the exact scale thresholds.
//
// Memory: one thread owns one 16-element block per step: one 32-byte load,
// one 8-byte code store, and one 4-byte store of four consecutive block scales
// per four lanes (gathered with shuffles).  HBM-bound: 2.5625 bytes/element.
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "fh_internal.h"

namespace fh {

namespace {

constexpr int kQuantThreads = 256;
constexpr uint32_t kBf16Inf = 0x7F80u;

// Exact positive E4M3 value of code c (1..126) in FP64.
__device__ __forceinline__ double e4m3_magnitude(int c) {
  const int e = c >> 3, m = c & 7;
  if (e == 0) return (double)m * 0x1p-9;
  // (8 + m) * 2^(e - 10), with the power of two built exactly.
  const double p2 = __longlong_as_double((long long)(1023 + e - 10) << 52);
  return (double)(8 + m) * p2;
}

// Smallest BF16 (as 16 magnitude bits) that is >= T (strict == false) or > T
// (strict == true), for T > 0; +Inf bits when no finite BF16 qualifies.
__device__ uint32_t bf16_threshold(double T, bool strict) {
  const float f = __double2float_ru(T);  // smallest FP32 >= T
  const uint32_t u = __float_as_uint(f);
  uint32_t r = (u > 0x7F7F0000u) ? 0x7F800000u : ((u + 0xFFFFu) & 0xFFFF0000u);
  if (strict && r != 0x7F800000u && (double)__uint_as_float(r) == T) r += 0x10000u;
  return r >> 16;
}

// E4M3 x2 conversion (round to nearest even, saturating); returns the low byte's code.
__device__ __forceinline__ uint32_t cvt_e4m3_sat(float v) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
  return r & 0xFFu;
}

// E2M1 x2 conversion: result bits 7..4 = code(hi), bits 3..0 = code(lo).
__device__ __forceinline__ uint32_t cvt_e2m1x2(float hi, float lo) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float bf16_to_float(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

// Fast-path code of one BF16 element at multiplier inv (4 bits with sign).
__device__ __forceinline__ uint32_t fast_code(uint32_t bits16, float inv) {
  return cvt_e2m1x2(0.0f, bf16_to_float(bits16) * inv) & 0xFu;
}

struct QuantTable {
  uint16_t scale_thr[128];    // [c]: smallest |amax| (BF16 bits) whose exact scale code is >= c
  uint16_t code_thr[128][8];  // [c][j<7]: smallest |x| whose exact magnitude code is >= j+1 at scale code c
  float inv[128];             // 1 / (S_c * s_g) for the converter path (0 for c == 0)
  uint32_t fast_ok[4];        // bit c: converter path verified exact at scale code c
};

// Exact magnitude code of |x| bits a at scale code c, from the table.
__device__ __forceinline__ uint32_t exact_mag(const QuantTable& t, int c, uint32_t a) {
  uint32_t m = 0;
#pragma unroll
  for (int j = 0; j < 7; ++j) m += (a >= t.code_thr[c][j]) ? 1u : 0u;
  return m;
}

__device__ void build_table(QuantTable& t, float sg_f) {
  const double sg = (double)sg_f;
  const double e2m1_mid[7] = {0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0};
  for (int i = threadIdx.x; i < 128 * 8; i += blockDim.x) {
    const int c = i >> 3, j = i & 7;
    if (j == 7) {
      uint32_t v;
      if (c == 0) {
        v = 0;
      } else if (c == 127) {
        v = kBf16Inf;  // sentinel: no amax reaches code 127 (NaN)
      } else {
        // Between codes c-1 and c; a tie goes to the even one.
        const double lo = (c == 1) ? 0.0 : e4m3_magnitude(c - 1);
        const double mid = 0.5 * (lo + e4m3_magnitude(c));
        v = bf16_threshold(mid * 6.0 * sg, ((c - 1) & 1) == 0);
      }
      t.scale_thr[c] = (uint16_t)v;
      t.code_thr[c][7] = (uint16_t)kBf16Inf;
    } else {
      uint32_t v = kBf16Inf;
      if (c != 0 && c != 127) {
        // Between magnitude codes j and j+1; a tie goes to the even one.
        v = bf16_threshold(e2m1_mid[j] * e4m3_magnitude(c) * sg, (j & 1) == 0);
      }
      t.code_thr[c][j] = (uint16_t)v;
    }
  }
  for (int c = threadIdx.x; c < 128; c += blockDim.x)
    t.inv[c] = (c == 0 || c == 127) ? 0.0f : (float)(1.0 / (e4m3_magnitude(c) * sg));
  if (threadIdx.x < 4) t.fast_ok[threadIdx.x] = (threadIdx.x == 3) ? 0x7FFFFFFFu : 0xFFFFFFFFu;
  __syncthreads();

  // Check the converter against the exact codes at both sides of every
  // decision boundary, at the ends of the BF16 range, and for both signs.
  for (int i = threadIdx.x; i < 127 * 8; i += blockDim.x) {
    const int c = i >> 3, j = i & 7;
    const float inv = t.inv[c];
    uint32_t probe[2];
    int np = 0;
    if (j < 7) {
      const uint32_t thr = t.code_thr[c][j];
      if (thr <= 0x7F7Fu) {
        probe[np++] = thr;
        if (thr > 0) probe[np++] = thr - 1;
      }
    } else {
      probe[np++] = 0;
      probe[np++] = 0x7F7Fu;
    }
    bool ok = true;
    for (int p = 0; p < np; ++p) {
      const uint32_t a = probe[p];
      const uint32_t want = exact_mag(t, c, a);
      ok = ok && (fast_code(a, inv) == want) && (fast_code(a | 0x8000u, inv) == (want | 8u));
    }
    if (!ok) atomicAnd(&t.fast_ok[c >> 5], ~(1u << (c & 31)));
  }
  __syncthreads();
}

// 16 BF16 values (8 words) -> 8 code bytes (2 words), exact-threshold path.
__device__ __forceinline__ void codes_exact(const QuantTable& t, int c, const uint32_t w[8],
                                            uint32_t out[2]) {
  uint32_t thr[7];
#pragma unroll
  for (int j = 0; j < 7; ++j) thr[j] = t.code_thr[c][j];
  out[0] = out[1] = 0;
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
}

// 16 BF16 values -> 8 code bytes via the converter at multiplier inv.
__device__ __forceinline__ void codes_fast(float inv, const uint32_t w[8], uint32_t out[2]) {
  uint32_t b[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float lo = __uint_as_float(w[i] << 16) * inv;
    const float hi = __uint_as_float(w[i] & 0xFFFF0000u) * inv;
    b[i] = cvt_e2m1x2(hi, lo);
  }
  out[0] = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
  out[1] = b[4] | (b[5] << 8) | (b[6] << 16) | (b[7] << 24);
}

__device__ __forceinline__ void load_block(const uint16_t* p, uint32_t w[8], bool wide) {
  if (wide) {
    asm volatile("ld.global.nc.L1::no_allocate.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]),
                   "=r"(w[6]), "=r"(w[7])
                 : "l"(p));
  } else {
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                 : "l"(p));
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7])
                 : "l"(p + 8));
  }
}

__device__ __forceinline__ int64_t tiled_offset(int64_t m, int64_t s, int64_t katoms) {
  return ((m >> 7) * katoms + (s >> 2)) * 512 + (m & 31) * 16 + ((m >> 5) & 3) * 4 + (s & 3);
}

// kGather4: K/16 % 4 == 0, so lanes 4i..4i+3 own four consecutive scales of
// one row and store them as one word.
template <bool kTiled, bool kGather4>
__global__ void __launch_bounds__(kQuantThreads) quantize_kernel(
    const uint16_t* __restrict__ x, int64_t M, int64_t K, int64_t ldx, float sg, float inv6sg,
    uint32_t clip_thr, bool wide, uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
    unsigned long long* __restrict__ clip_count) {
  __shared__ QuantTable tab;
  __shared__ unsigned long long cta_clips;
  if (threadIdx.x == 0) cta_clips = 0;
  build_table(tab, sg);

  const int lane = threadIdx.x & 31;
  const int64_t nb = K >> 4;
  const int64_t total = M * nb;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t katoms = nb >> 2;
  const int64_t dm = stride / nb, ds = stride % nb;
  int64_t base = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31);
  int64_t b = base + lane;
  int64_t m = b / nb, s = b % nb;
  unsigned long long clips = 0;

  for (; base < total; base += stride) {
    const bool valid = b < total;
    uint32_t w[8];
    uint32_t sc = 0;
    if (valid) {
      load_block(x + m * ldx + 16 * s, w, wide);
      // Block amax over the 15 magnitude bits of each BF16.
      uint32_t mx = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        uint32_t r;
        asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(mx), "r"(w[i] & 0x7FFF7FFFu));
        mx = r;
      }
      const uint32_t amax = max(mx & 0xFFFFu, mx >> 16);
      // Scale code: converter candidate, corrected against the exact thresholds.
      const float amax_f = bf16_to_float(amax);
      uint32_t c = min(cvt_e4m3_sat(amax_f * inv6sg), 126u);
      while (c < 126u && amax >= tab.scale_thr[c + 1]) ++c;
      while (c > 0u && amax < tab.scale_thr[c]) --c;
      sc = c;
      // Element codes.
      uint32_t out[2];
      const float inv = tab.inv[c];
      const bool fast = ((tab.fast_ok[c >> 5] >> (c & 31)) & 1u) && (amax_f * inv <= 3.0e38f);
      if (fast)
        codes_fast(inv, w, out);
      else
        codes_exact(tab, (int)c, w, out);
      *reinterpret_cast<uint2*>(codes + m * (K >> 1) + 8 * s) = make_uint2(out[0], out[1]);
      // Clipped elements: only blocks whose amax is beyond the limit have any.
      if (amax >= clip_thr) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          clips += ((w[i] & 0x7FFFu) >= clip_thr) ? 1u : 0u;
          clips += (((w[i] >> 16) & 0x7FFFu) >= clip_thr) ? 1u : 0u;
        }
      }
    }
    if (kGather4) {
      const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, sc, 1);
      const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, sc, 2);
      const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, sc, 3);
      if (valid && (lane & 3) == 0) {
        const uint32_t word = sc | (s1 << 8) | (s2 << 16) | (s3 << 24);
        const int64_t off = kTiled ? tiled_offset(m, s, katoms) : m * nb + s;
        *reinterpret_cast<uint32_t*>(scales + off) = word;
      }
    } else if (valid) {
      scales[kTiled ? tiled_offset(m, s, katoms) : m * nb + s] = (uint8_t)sc;
    }
    b += stride;
    s += ds;
    m += dm;
    if (s >= nb) {
      s -= nb;
      ++m;
    }
  }

  if (kTiled) {
    // Zero the scales of the padding rows M .. ceil(M/128)*128 - 1.
    const int64_t mpad = ((M + 127) >> 7) << 7;
    const int64_t npad = (mpad - M) * nb;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < npad; i += stride) {
      const int64_t pm = M + i / nb, ps = i % nb;
      scales[tiled_offset(pm, ps, katoms)] = 0;
    }
  }

  // Clip count: warp sum, CTA sum, one atomic per CTA that saw any.
  unsigned long long wsum = clips;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xFFFFFFFFu, wsum, o);
  if (lane == 0 && wsum) atomicAdd(&cta_clips, wsum);
  __syncthreads();
  if (threadIdx.x == 0 && cta_clips && clip_count) atomicAdd(clip_count, cta_clips);
}

// ---------------------------------------------------------------------------
// Calibration amax
// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(256) amax_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                   int64_t cols, int64_t ldx, bool vec,
                                                   float* __restrict__ out) {
  uint32_t mx = 0;  // max magnitude bits
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (vec) {
    const int64_t cpr = cols >> 3;  // 8-element chunks per row
    const int64_t total = rows * cpr;
    for (int64_t i = tid; i < total; i += stride) {
      const int64_t r = i / cpr, ch = i % cpr;
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(x + r * ldx + 8 * ch));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        uint32_t t;
        asm("max.u16x2 %0, %1, %2;" : "=r"(t) : "r"(mx), "r"(w[k] & 0x7FFF7FFFu));
        mx = t;
      }
    }
    mx = max(mx & 0xFFFFu, mx >> 16);
  } else {
    const int64_t total = rows * cols;
    for (int64_t i = tid; i < total; i += stride) {
      const int64_t r = i / cols, c = i % cols;
      mx = max(mx, (uint32_t)(x[r * ldx + c] & 0x7FFFu));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
  __shared__ uint32_t red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 1; i < (int)(blockDim.x >> 5); ++i) mx = max(mx, red[i]);
    // Non-negative floats order like their bit patterns.
    atomicMax(reinterpret_cast<unsigned int*>(out), mx << 16);
  }
}

// ---------------------------------------------------------------------------
// Scale relayout and GELU
// ---------------------------------------------------------------------------

__global__ void scales_to_rowmajor_kernel(const uint8_t* __restrict__ tiled,
                                          uint8_t* __restrict__ rowmajor, int64_t rows,
                                          int64_t K) {
  const int64_t nb = K >> 4, katoms = nb >> 2;
  const int64_t total = rows * nb;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / nb, s = i % nb;
    rowmajor[i] = tiled[tiled_offset(r, s, katoms)];
  }
}

__device__ __forceinline__ uint32_t gelu_bits(uint32_t bits16) {
  const float v = bf16_to_float(bits16);
  const float y = 0.5f * v * (1.0f + erff(v * 0.70710678118654752440f));
  return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(y));
}

__global__ void gelu_kernel(const uint16_t* __restrict__ x, uint16_t* __restrict__ y, int64_t n) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t nvec = n >> 3;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nvec; i += stride) {
    uint4 v = reinterpret_cast<const uint4*>(x)[i];
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) w[k] = gelu_bits(w[k] & 0xFFFFu) | (gelu_bits(w[k] >> 16) << 16);
    reinterpret_cast<uint4*>(y)[i] = make_uint4(w[0], w[1], w[2], w[3]);
  }
  for (int64_t i = (nvec << 3) + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
    y[i] = (uint16_t)gelu_bits(x[i]);
}

int grid_for(int64_t work_items, int threads, int per_sm) {
  const int64_t want = (work_items + threads - 1) / threads;
  const int64_t cap = (int64_t)sm_count() * per_sm;
  return (int)(want < 1 ? 1 : (want < cap ? want : cap));
}

}  // namespace

cudaError_t launch_quantize(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, float sg,
                            uint8_t* codes, uint8_t* scales, unsigned long long* clip,
                            int layout, cudaStream_t s) {
  const int64_t nb = K / 16;
  const bool tiled = layout == FH_SCALES_MMA_TILED;
  const bool gather4 = (nb % 4) == 0;
  const bool wide = ((reinterpret_cast<uintptr_t>(x) & 31) == 0) && ((ldx % 16) == 0);
  // Exact clip threshold: smallest BF16 magnitude strictly beyond 2688 * s_g
  // (2688 * s_g is exact in FP64: 5 + 24 significant bits).
  const double limit = 2688.0 * (double)sg;
  uint32_t clip_thr;
  {
    float f = (float)limit;
    if ((double)f < limit) f = nextafterf(f, INFINITY);  // smallest FP32 >= limit
    uint32_t u;
    memcpy(&u, &f, 4);
    if (u > 0x7F7F0000u) {
      clip_thr = 0x7F80u;
    } else {
      uint32_t r = (u + 0xFFFFu) & 0xFFFF0000u;  // smallest BF16 >= limit
      float rf;
      memcpy(&rf, &r, 4);
      if ((double)rf == limit) r += 0x10000u;  // strictly beyond
      clip_thr = r >> 16;
    }
  }
  const float inv6sg = (float)(1.0 / (6.0 * (double)sg));
  const int64_t mpad = tiled ? ((M + 127) / 128) * 128 : M;
  const int grid = grid_for((mpad > M ? mpad : M) * nb, kQuantThreads, 8);
  if (tiled) {
    if (gather4)
      quantize_kernel<true, true><<<grid, kQuantThreads, 0, s>>>(x, M, K, ldx, sg, inv6sg, clip_thr,
                                                                 wide, codes, scales, clip);
    else
      quantize_kernel<true, false><<<grid, kQuantThreads, 0, s>>>(x, M, K, ldx, sg, inv6sg, clip_thr,
                                                                  wide, codes, scales, clip);
  } else {
    if (gather4)
      quantize_kernel<false, true><<<grid, kQuantThreads, 0, s>>>(x, M, K, ldx, sg, inv6sg, clip_thr,
                                                                  wide, codes, scales, clip);
    else
      quantize_kernel<false, false><<<grid, kQuantThreads, 0, s>>>(x, M, K, ldx, sg, inv6sg,
                                                                   clip_thr, wide, codes, scales, clip);
  }
  return cudaGetLastError();
}

cudaError_t launch_amax(const uint16_t* x, int64_t rows, int64_t cols, int64_t ldx, float* amax,
                        cudaStream_t s) {
  const bool vec = (cols % 8 == 0) && (ldx % 8 == 0) && ((reinterpret_cast<uintptr_t>(x) & 15) == 0);
  const int grid = grid_for(vec ? rows * (cols / 8) : rows * cols, 256, 8);
  amax_kernel<<<grid, 256, 0, s>>>(x, rows, cols, ldx, vec, amax);
  return cudaGetLastError();
}

cudaError_t launch_scales_to_rowmajor(const uint8_t* tiled, uint8_t* rowmajor, int64_t rows,
                                      int64_t K, cudaStream_t s) {
  const int grid = grid_for(rows * (K / 16), 256, 8);
  scales_to_rowmajor_kernel<<<grid, 256, 0, s>>>(tiled, rowmajor, rows, K);
  return cudaGetLastError();
}

cudaError_t launch_gelu(const uint16_t* x, uint16_t* y, int64_t n, cudaStream_t s) {
  const int grid = grid_for((n + 7) / 8, 256, 8);
  gelu_kernel<<<grid, 256, 0, s>>>(x, y, n);
  return cudaGetLastError();
}

}  // namespace fh
