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
// BF16 at (or beyond) the threshold.  For a given s_g the host builds, in FP64
// (where t * S * s_g is exact), these BF16 decision thresholds for all 126
// finite non-zero scale codes, once per distinct s_g (cached), and passes them
// to the kernel as a parameter; each CTA copies the 2.8 KB table to shared
// memory.  Elements then go through the hardware converter on x * (1/(S s_g))
// -- one multiply per element, two elements per cvt -- but only for scale
// codes where the host has checked, at both sides of every decision boundary,
// that the converter's documented rounding (round to nearest even, saturating
// to the largest finite value) of that FP32 product gives the exact code; the
// multiply and the converter are monotone, so agreement at every boundary
// means agreement on every BF16 input.  Blocks whose scale code failed the
// check (exact ties at non-power-of-two scales, typically) take the exact
// threshold-compare path.  The block scale takes a converter candidate and
// corrects it against the exact scale thresholds.
//
// Memory: a producer warp streams units of x into a 96 KB ring of
// shared-memory stages; each of 512 consumer threads quantizes one 16-element
// block per 64 columns of the unit (one 32-byte shared-memory read, one 8-byte
// code store).  For the tensor-core scale layout a unit is a 128-row x
// 128-column tile (128 x 64 when K is an odd multiple of 64), whose whole
// 512-byte scale atoms are staged in shared memory and copied out by the
// producer warp; for row-major scales a unit is whole rows of 16 KB and four
// lanes gather four consecutive block scales into one 4-byte store.
// HBM-bound: 2.5625 bytes per element.
#include <cuda_bf16.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "fh_internal.h"
#include "fh_nvfp4.cuh"

namespace fh {

namespace {

constexpr uint32_t kBf16Inf = 0x7F80u;

using namespace nvfp4;

struct QuantParams {
  QuantTable tab;
  const uint16_t* x;
  uint8_t* codes;
  uint8_t* scales;
  unsigned long long* clip;
  int64_t M, K, ldx;
  float inv6sg;       // 1 / (6 s_g): scale-code candidate multiplier
  uint32_t clip_thr;  // smallest BF16 magnitude strictly beyond 2688 s_g
  // Streaming units: R rows x kc columns (kc divides K), at most 8192 elements.
  int64_t kc, R, col_units, n_units;
  int nbu;            // 16-element blocks per unit row: kc / 16
  int step_rows;      // consumer stride in blocks (256) as whole rows ...
  int step_blocks;    // ... plus remaining blocks: 256 = step_rows * nbu + step_blocks
  int one_copy;       // rows of a unit are contiguous in x: one bulk copy per unit
};

// ---- host: the exact decision table for one global scale ----------------------

// Exact positive E4M3 value of code c (1..126).
double e4m3_magnitude(int c) {
  const int e = c >> 3, m = c & 7;
  return e == 0 ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10);
}

// Smallest BF16 (16 magnitude bits) >= T, or > T when strict, for T > 0;
// +Inf bits when no finite BF16 qualifies.
uint32_t bf16_threshold(double T, bool strict) {
  float f = (float)T;
  if ((double)f < T) f = nextafterf(f, INFINITY);  // smallest FP32 >= T
  uint32_t u;
  memcpy(&u, &f, 4);
  uint32_t r = (u > 0x7F7F0000u) ? 0x7F800000u : ((u + 0xFFFFu) & 0xFFFF0000u);
  if (strict && r != 0x7F800000u) {
    float rf;
    memcpy(&rf, &r, 4);
    if ((double)rf == T) r += 0x10000u;
  }
  return r >> 16;
}

float bf16_bits_value(uint32_t bits16) {
  const uint32_t u = bits16 << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

// The converter's documented result on a magnitude y >= 0: nearest E2M1 grid
// point, ties to the even code, saturating at 6 (Inf included).
uint32_t converter_e2m1(float y) {
  static const float grid[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
  if (!(y < 6.0f)) return 7;
  uint32_t c = 0;
  for (int k = 1; k < 8; ++k) {
    const float mid = 0.5f * (grid[k - 1] + grid[k]);
    if (y > mid || (y == mid && (k & 1) == 0)) c = (uint32_t)k;
  }
  return c;
}

void build_table(float sg_f, QuantTable* t) {
  const double sg = (double)sg_f;
  static const double e2m1_mid[7] = {0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0};
  memset(t, 0, sizeof *t);
  uint16_t scale_thr[128];  // [c]: smallest block amax (BF16 bits) whose exact scale code is >= c
  float inv[128];           // 1 / (S_c * s_g): multiplier of the converter path (0 for c == 0)
  bool fast_ok[128] = {};   // the converter path is exact at scale code c
  for (int c = 0; c < 128; ++c) {
    // Block scale: codes c-1 and c meet at their midpoint; a tie goes to the even code.
    if (c == 0) {
      scale_thr[c] = 0;
    } else if (c == 127) {
      scale_thr[c] = (uint16_t)kBf16Inf;  // NaN code: never chosen
    } else {
      const double lo = (c == 1) ? 0.0 : e4m3_magnitude(c - 1);
      const double mid = 0.5 * (lo + e4m3_magnitude(c));
      scale_thr[c] = (uint16_t)bf16_threshold(mid * 6.0 * sg, ((c - 1) & 1) == 0);
    }
    // Element codes at scale code c: magnitude codes j and j+1 meet at the grid
    // midpoint times S_c * s_g; a tie goes to the even code.
    for (int j = 0; j < 8; ++j) {
      uint32_t v = kBf16Inf;
      if (j < 7 && c != 0 && c != 127)
        v = bf16_threshold(e2m1_mid[j] * e4m3_magnitude(c) * sg, (j & 1) == 0);
      t->code_thr[c][j] = (uint16_t)v;
    }
    inv[c] = (c == 0 || c == 127) ? 0.0f : (float)(1.0 / (e4m3_magnitude(c) * sg));
  }
  // Converter path check at both sides of every boundary and at the ends of the
  // BF16 range.  Negative inputs give the same magnitude with the sign bit set.
  // When the FP32 product of a boundary value lands on a midpoint the nearest
  // multiplier fails the check; a neighbouring FP32 multiplier usually passes,
  // so up to two on each side are tried before the code falls back to the
  // exact threshold path.
  for (int c = 0; c < 127; ++c) {
    auto exact_mag = [&](uint32_t a) {
      uint32_t m = 0;
      for (int j = 0; j < 7; ++j) m += (a >= t->code_thr[c][j]) ? 1u : 0u;
      return m;
    };
    auto passes = [&](float inv) {
      bool ok = true;
      auto probe = [&](uint32_t a) {
        const float y = bf16_bits_value(a) * inv;  // the kernel's FP32 multiply
        ok = ok && converter_e2m1(y) == exact_mag(a);
      };
      probe(0);
      probe(0x7F7Fu);
      for (int j = 0; j < 7; ++j) {
        const uint32_t thr = t->code_thr[c][j];
        if (thr <= 0x7F7Fu) {
          probe(thr);
          if (thr > 0) probe(thr - 1);
        }
      }
      return ok;
    };
    const float inv0 = inv[c];
    const float up1 = nextafterf(inv0, INFINITY), dn1 = nextafterf(inv0, 0.0f);
    const float cand[5] = {inv0, up1, dn1, nextafterf(up1, INFINITY), nextafterf(dn1, 0.0f)};
    for (float m : cand) {
      if (passes(m)) {
        inv[c] = m;
        fast_ok[c] = true;
        break;
      }
    }
  }
  // The packed per-code entries the kernels read.
  for (int c = 0; c < 128; ++c) {
    uint32_t bits;
    memcpy(&bits, &inv[c], 4);
    const uint32_t next = (c < 127) ? scale_thr[c + 1] : kBf16Inf;
    t->sc[c] = make_uint2(bits, (uint32_t)scale_thr[c] | (fast_ok[c] ? 0x8000u : 0u) | (next << 16));
  }
}

}  // namespace

// Small per-thread cache: calibrated layers reuse one s_g for every call.
const QuantTable& quant_table_for(float sg) {
  struct Entry {
    float sg;
    bool valid;
    QuantTable t;
  };
  thread_local Entry cache[4] = {};
  thread_local int next = 0;
  for (auto& e : cache)
    if (e.valid && e.sg == sg) return e.t;
  Entry& e = cache[next];
  next = (next + 1) & 3;
  build_table(sg, &e.t);
  e.sg = sg;
  e.valid = true;
  return e.t;
}

uint32_t clip_threshold_bits(float sg) { return bf16_threshold(2688.0 * (double)sg, true); }

namespace {

// ---- device --------------------------------------------------------------------

__device__ __forceinline__ int64_t tiled_offset(int64_t m, int64_t s, int64_t katoms) {
  return ((m >> 7) * katoms + (s >> 2)) * 512 + (m & 31) * 16 + ((m >> 5) & 3) * 4 + (s & 3);
}

// Quantize one loaded block: stores its 8 code bytes at dst, returns its scale
// code and adds its clipped elements to clips.
__device__ __forceinline__ uint32_t quantize_block_to(const QuantTable& tab, const QuantParams& p,
                                                      const uint32_t* w, uint8_t* dst,
                                                      unsigned long long& clips) {
  uint32_t amax;
  uint2 out;
  const uint32_t c = quantize_block_codes(tab, p.inv6sg, w, amax, out);
  *reinterpret_cast<uint2*>(dst) = out;
  clips += block_clips(w, amax, p.clip_thr);
  return c;
}

// Quantize one loaded block of row m: stores its 8 code bytes, returns its
// scale code and adds its clipped elements to clips.
__device__ __forceinline__ uint32_t quantize_block(const QuantTable& tab, const QuantParams& p,
                                                   const uint32_t* w, int64_t m, int64_t s,
                                                   unsigned long long& clips) {
  uint32_t amax;
  uint2 out;
  const uint32_t c = quantize_block_codes(tab, p.inv6sg, w, amax, out);
  *reinterpret_cast<uint2*>(p.codes + m * (p.K >> 1) + 8 * s) = out;
  clips += block_clips(w, amax, p.clip_thr);
  return c;
}

template <bool kTiled, bool kGather4>
__device__ __forceinline__ void store_scale(const QuantParams& p, uint32_t sc, bool valid, int lane, int64_t m,
                                            int64_t s, int64_t nb, int64_t katoms) {
  if (kGather4) {
    // Lanes 4i..4i+3 hold four consecutive scales of one row.
    const uint32_t pair = sc | (__shfl_down_sync(0xFFFFFFFFu, sc, 1) << 8);
    const uint32_t word = pair | (__shfl_down_sync(0xFFFFFFFFu, pair, 2) << 16);
    if (valid && (lane & 3) == 0)
      *reinterpret_cast<uint32_t*>(p.scales + (kTiled ? tiled_offset(m, s, katoms) : m * nb + s)) = word;
  } else if (valid) {
    p.scales[kTiled ? tiled_offset(m, s, katoms) : m * nb + s] = (uint8_t)sc;
  }
}

// Streaming layout of the quantizer: one producer warp moves units of 8192 BF16
// elements (16 KB) from HBM into a ring of shared-memory stages with
// asynchronous bulk or tensor copies; sixteen consumer warps quantize each unit
// from shared memory, one 16-element block per thread.  Two CTAs per SM keep
// ~190 KB of loads in flight per SM.
constexpr int kQConsumerWarps = 16;
constexpr int kQThreads = 32 * (kQConsumerWarps + 1);
constexpr int kQStages = 6;
constexpr int kQUnitElems = 8192;
constexpr int kQUnitBytes = 2 * kQUnitElems;
// The tiled kernel stages each unit's scale atoms in shared memory (two
// buffers per ring stage); the producer warp copies them out.
constexpr int kQScaleStaging = 2 * kQStages * 512;
constexpr int kQSmem = kQStages * kQUnitBytes + kQScaleStaging + 2 * 8 * kQStages + 64;
static_assert(kQUnitElems / 16 == 32 * kQConsumerWarps, "one block per consumer thread per unit");

__device__ unsigned int g_quant_error = 0;

__device__ __forceinline__ uint32_t q_smem_u32(const void* ptr) { return (uint32_t)__cvta_generic_to_shared(ptr); }

__device__ __forceinline__ bool q_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// L2 policy of the loads of x: every byte of x is read exactly once, so its
// lines are the first candidates for eviction.  Lines that other kernels left
// in L2 -- notably the preceding GEMM's output, still dirty -- then stay there
// instead of being written back while this kernel streams x; their write-back
// happens later, under the next GEMM, which leaves HBM bandwidth to spare.
__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// Bounded wait (about 4 s, or until another warp of the CTA gave up).
__device__ __forceinline__ bool q_wait(uint32_t bar, uint32_t parity, volatile int* abort) {
  if (q_try_wait(bar, parity)) return true;
  uint64_t t0;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  for (uint32_t i = 1; i < (1u << 30); ++i) {
    if (q_try_wait(bar, parity)) return true;
    if ((i & 255u) == 0u) {
      if (*abort) return false;
      uint64_t t;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
      if (t - t0 > 4000000000ull) break;
    }
  }
  atomicOr(&g_quant_error, 1u);
  *abort = 1;
  return false;
}

// Wait used by the producer's drain: its copies must have landed before the
// CTA retires, so this ignores the abort flag and gives up only on its own
// time limit (~1 s).
__device__ __forceinline__ void q_wait_drain(uint32_t bar, uint32_t parity) {
  if (q_try_wait(bar, parity)) return;
  uint64_t t0;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  for (uint32_t i = 1; i < (1u << 30); ++i) {
    if (q_try_wait(bar, parity)) return;
    if ((i & 255u) == 0u) {
      uint64_t t;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
      if (t - t0 > 1000000000ull) break;
    }
  }
  atomicOr(&g_quant_error, 1u);
}

// Row-major scale layout.  kGather4: K/16 % 4 == 0, so lanes 4i..4i+3 own four
// consecutive scales of one row and store them as one word.
template <bool kGather4>
__global__ void __launch_bounds__(kQThreads) quantize_kernel(const __grid_constant__ QuantParams p) {
  extern __shared__ __align__(128) uint8_t qsmem[];
  __shared__ QuantTable tab;
  __shared__ unsigned long long cta_clips;
  __shared__ int abort_flag_s;
  volatile int* abort_flag = &abort_flag_s;
  const uint32_t stage0 = q_smem_u32(qsmem);
  const uint32_t bar0 = stage0 + kQStages * kQUnitBytes;
  auto full_bar = [&](int st) { return bar0 + 8u * st; };
  auto empty_bar = [&](int st) { return bar0 + 8u * (kQStages + st); };
  {
    const uint4* src = reinterpret_cast<const uint4*>(&p.tab);
    uint4* dst = reinterpret_cast<uint4*>(&tab);
    for (int i = threadIdx.x; i < (int)(sizeof(QuantTable) / 16); i += blockDim.x) dst[i] = src[i];
  }
  if (threadIdx.x == 0) {
    cta_clips = 0;
    abort_flag_s = 0;
    for (int st = 0; st < kQStages; ++st) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(full_bar(st)));
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(empty_bar(st)), "r"(kQConsumerWarps));
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nb = p.K >> 4;
  const int64_t katoms = nb >> 2;
  unsigned long long clips = 0;

  if (warp == kQConsumerWarps) {
    // ===== producer: bulk copies of whole units into the stage ring =====
    if (lane == 0) {
      const uint64_t read_once = evict_first_policy();
      int st = 0;
      uint32_t ph = 0;
      for (int64_t u = blockIdx.x; u < p.n_units; u += gridDim.x) {
        if (!q_wait(empty_bar(st), ph ^ 1u, abort_flag)) break;
        const int64_t rb = p.col_units == 1 ? u : u / p.col_units;
        const int64_t cb = p.col_units == 1 ? 0 : u % p.col_units;
        const int64_t r0 = rb * p.R;
        const int64_t rows = min(p.R, p.M - r0);
        const uint32_t row_bytes = (uint32_t)(p.kc * 2);
        const uint32_t dst = stage0 + st * kQUnitBytes;
        const uint16_t* src = p.x + r0 * p.ldx + cb * p.kc;
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(full_bar(st)),
                     "r"((uint32_t)rows * row_bytes)
                     : "memory");
        if (p.one_copy) {
          asm volatile(
              "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
              " [%0], [%1], %2, [%3], %4;" ::"r"(dst),
              "l"(src), "r"((uint32_t)rows * row_bytes), "r"(full_bar(st)), "l"(read_once)
              : "memory");
        } else {
          for (int64_t r = 0; r < rows; ++r)
            asm volatile(
                "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
                " [%0], [%1], %2, [%3], %4;" ::"r"(dst + (uint32_t)r * row_bytes),
                "l"(src + r * p.ldx), "r"(row_bytes), "r"(full_bar(st)), "l"(read_once)
                : "memory");
        }
        if (++st == kQStages) {
          st = 0;
          ph ^= 1u;
        }
      }
      // Drain: every copy this thread issued has landed before the CTA retires.
      for (int i = 0; i < kQStages; ++i) q_wait_drain(full_bar(i), (i < st) ? ph : (ph ^ 1u));
    }
  } else {
    // ===== consumers: thread t quantizes block t of every unit =====
    const int ctid = threadIdx.x;  // 0 .. 511
    const int64_t ublocks = p.R * p.nbu;  // blocks in a full unit
    const int r = ctid / p.nbu, sb = ctid % p.nbu;  // the same place in every unit
    const bool in_unit = ctid < ublocks;
    const uint8_t* my_block = qsmem + 32 * ctid;
    int st = 0;
    uint32_t ph = 0;
    for (int64_t u = blockIdx.x; u < p.n_units; u += gridDim.x) {
      if (!q_wait(full_bar(st), ph, abort_flag)) break;
      const int64_t rb = p.col_units == 1 ? u : u / p.col_units;
      const int64_t cb = p.col_units == 1 ? 0 : u % p.col_units;
      const int64_t m = rb * p.R + r;
      const int64_t sg = cb * p.nbu + sb;  // block index within the row
      const bool valid = in_unit && (m < p.M);
      uint32_t sc = 0;
      if (valid) {
        const uint8_t* blk = my_block + st * kQUnitBytes;
        const uint4 q0 = *reinterpret_cast<const uint4*>(blk);
        const uint4 q1 = *reinterpret_cast<const uint4*>(blk + 16);
        const uint32_t w[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
        sc = quantize_block(tab, p, w, m, sg, clips);
      }
      store_scale<false, kGather4>(p, sc, valid, lane, m, sg, nb, katoms);
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(empty_bar(st)) : "memory");
      if (++st == kQStages) {
        st = 0;
        ph ^= 1u;
      }
    }
  }

  // Clip count: warp sum, CTA sum, one atomic per CTA that saw any.
  unsigned long long wsum = clips;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xFFFFFFFFu, wsum, o);
  if (lane == 0 && wsum) atomicAdd(&cta_clips, wsum);
  __syncthreads();
  if (threadIdx.x == 0 && cta_clips && p.clip) atomicAdd(p.clip, cta_clips);
}

// Tensor-core scale layout: each unit is a 128-row x 64 kG-column tile of x
// (16 kG KB), loaded by one 2-D tensor TMA whose out-of-range rows read as
// zero.  Thread t quantizes block t % 4 of every 64-column group of tile row
// t / 4, so one unit yields exactly kG whole 512-byte scale atoms and 32-byte
// code segments; zero rows past M give the zero padding scales the layout
// requires.  The consumers leave each scale byte in a shared-memory staging
// buffer, and the producer warp, once the unit's stage is released, copies
// the unit's atoms out with 16-byte stores (one scale store per lane instead
// of gathers and a 4-byte store per row).  The wider unit halves the TMA
// issues and barrier round trips per byte; the ring keeps the same 96 KB.
// kGelu: quantize GELU(x) instead of x (the FFN activation applied on the way,
// with the same arithmetic as the stand-alone GELU kernel).
template <bool kGelu, int kG>
__global__ void __launch_bounds__(kQThreads) quantize_tiled_kernel(const __grid_constant__ CUtensorMap tmx,
                                                                   const __grid_constant__ QuantParams p) {
  // A unit is 128 rows x 64 kG columns (kG scale atoms); the ring holds the
  // same 96 KB for either width.
  constexpr int S = kQStages / kG;
  constexpr int kUnitBytes = kQUnitBytes * kG;
  extern __shared__ __align__(128) uint8_t qsmem[];
  __shared__ QuantTable tab;
  __shared__ unsigned long long cta_clips;
  __shared__ int abort_flag_s;
  volatile int* abort_flag = &abort_flag_s;
  const uint32_t stage0 = q_smem_u32(qsmem);
  // Scale staging: buffer (st, b) holds the kG atoms of the unit in ring stage
  // st whose ring phase bit is b.
  const uint32_t sstage0 = stage0 + S * kUnitBytes;
  auto scale_buf = [&](int st, uint32_t b) { return sstage0 + (uint32_t)((2 * st + (int)b) * kG * 512); };
  const uint32_t bar0 = sstage0 + kQScaleStaging;
  auto full_bar = [&](int st) { return bar0 + 8u * st; };
  auto empty_bar = [&](int st) { return bar0 + 8u * (S + st); };
  static_assert(2 * S * kG * 512 == kQScaleStaging, "staging size");
  {
    const uint4* src = reinterpret_cast<const uint4*>(&p.tab);
    uint4* dst = reinterpret_cast<uint4*>(&tab);
    for (int i = threadIdx.x; i < (int)(sizeof(QuantTable) / 16); i += blockDim.x) dst[i] = src[i];
  }
  if (threadIdx.x == 0) {
    cta_clips = 0;
    abort_flag_s = 0;
    for (int st = 0; st < S; ++st) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(full_bar(st)));
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(empty_bar(st)), "r"(kQConsumerWarps));
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmx)) : "memory");
  }
  __syncthreads();
  // A kernel launched as this one's programmatic dependent (the GEMM that
  // reads its output) may start its setup now; it waits for this grid to
  // complete before it reads anything.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nb = p.K >> 4;
  const int64_t katoms = nb >> 2;  // 64-column tiles (scale atoms) per row block
  unsigned long long clips = 0;
  // Unit u is tile (u / ka, u % ka) of ka = K / (64 kG) units per row block;
  // the CTA visits u = blockIdx.x, blockIdx.x + gridDim.x, ..., so both
  // coordinates advance by constants (no division inside the loops).
  const int ka = (int)katoms / kG;
  const int d_row = (int)(gridDim.x / ka), d_col = (int)(gridDim.x % ka);
  const int row0 = (int)(blockIdx.x / ka), col0 = (int)(blockIdx.x % ka);

  if (warp == kQConsumerWarps) {
    // ===== producer: one tensor TMA per 128 x 64 kG tile =====
    {
      const uint64_t read_once = evict_first_policy();
      int st = 0;
      uint32_t ph = 0;
      int tr = row0, tc = col0;  // the next unit to load
      int sr = row0, sc = col0;  // the next unit whose scales go out
      int64_t n = 0;             // units loaded
      bool ok = true;
      // Once the consumers are done with unit n - S (the wait for its ring
      // stage), the warp copies its staged scale atoms (kG x 512 contiguous
      // bytes) to global memory, 16 bytes per lane per step.
      auto store_scales = [&](int stage, uint32_t b) {
        const uint4* src = reinterpret_cast<const uint4*>(qsmem + (scale_buf(stage, b) - stage0));
        uint4* dst = reinterpret_cast<uint4*>(p.scales + ((int64_t)sr * katoms + (int64_t)sc * kG) * 512);
#pragma unroll
        for (int i = 0; i < kG; ++i) dst[32 * i + lane] = src[32 * i + lane];
        sr += d_row;
        sc += d_col;
        if (sc >= ka) {
          sc -= ka;
          ++sr;
        }
      };
      for (int64_t u = blockIdx.x; u < p.n_units; u += gridDim.x, ++n) {
        if (!__all_sync(0xFFFFFFFFu, q_wait(empty_bar(st), ph ^ 1u, abort_flag))) {  // warp-uniform
          ok = false;
          break;
        }
        // Staging buffer (st, ph ^ 1) held unit n - S; buffer (st, ph), which
        // unit n's consumers fill, was copied out S units ago.
        if (n >= S) store_scales(st, ph ^ 1u);
        const int x0 = tc * 64 * kG, y0 = tr * 128;
        tr += d_row;
        tc += d_col;
        if (tc >= ka) {
          tc -= ka;
          ++tr;
        }
        if (lane == 0) {
          asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(full_bar(st)),
                       "r"((uint32_t)kUnitBytes)
                       : "memory");
          asm volatile(
              "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
              " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(stage0 + st * kUnitBytes),
              "l"(reinterpret_cast<uint64_t>(&tmx)), "r"(x0), "r"(y0), "r"(full_bar(st)), "l"(read_once)
              : "memory");
        }
        __syncwarp();
        if (++st == S) {
          st = 0;
          ph ^= 1u;
        }
      }
      // The scales of the last S units, as their stages are released: the
      // ring walk continues over S more positions without loading.
      int tst = st;
      uint32_t tph = ph;
      for (int64_t k = n; ok && k < n + S; ++k) {
        if (!__all_sync(0xFFFFFFFFu, q_wait(empty_bar(tst), tph ^ 1u, abort_flag))) break;
        if (k >= S) store_scales(tst, tph ^ 1u);
        if (++tst == S) {
          tst = 0;
          tph ^= 1u;
        }
      }
      // The last load into each stage, from the position after the last loaded unit.
      if (lane == 0)
        for (int i = 0; i < S; ++i) q_wait_drain(full_bar(i), (i < st) ? ph : (ph ^ 1u));
      __syncwarp();
    }
  } else {
    // ===== consumers: thread t quantizes block t % 4 of every 64-column group of tile row t / 4 =====
    const int ctid = threadIdx.x;  // 0 .. 511
    const int r = ctid >> 2, j = ctid & 3;
    const uint8_t* my_block = qsmem + r * (128 * kG) + 32 * j;
    const uint32_t scale_off = (uint32_t)((r & 31) * 16 + (r >> 5) * 4 + j);  // this block's byte in an atom
    int st = 0;
    uint32_t ph = 0;
    int tr = row0, tc = col0;
    for (int64_t u = blockIdx.x; u < p.n_units; u += gridDim.x) {
      if (!q_wait(full_bar(st), ph, abort_flag)) break;
      const int64_t m = (int64_t)tr * 128 + r;
      const int cg0 = tc * kG;  // the unit's first 64-column group
      uint8_t* crow = p.codes + m * (p.K >> 1) + 32 * cg0 + 8 * j;
      const uint32_t sbuf = scale_buf(st, ph) + scale_off;
      tr += d_row;
      tc += d_col;
      if (tc >= ka) {
        tc -= ka;
        ++tr;
      }
#pragma unroll 1
      for (int c = 0; c < kG; ++c) {
        uint32_t sc = 0;
        if (m < p.M) {
          const uint8_t* blk = my_block + st * kUnitBytes + c * 128;
          const uint4 q0 = *reinterpret_cast<const uint4*>(blk);
          const uint4 q1 = *reinterpret_cast<const uint4*>(blk + 16);
          uint32_t w[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
          if (kGelu) {
#pragma unroll
            for (int i = 0; i < 8; ++i) w[i] = gelu2_bits(w[i]);
          }
          sc = quantize_block_to(tab, p, w, crow + 32 * c, clips);
        }
        // Every row of the unit, padding rows included, stages its scales.
        asm volatile("st.shared.u8 [%0], %1;" ::"r"(sbuf + 512u * c), "r"(sc) : "memory");
      }
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(empty_bar(st)) : "memory");
      if (++st == S) {
        st = 0;
        ph ^= 1u;
      }
    }
  }

  unsigned long long wsum = clips;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xFFFFFFFFu, wsum, o);
  if (lane == 0 && wsum) atomicAdd(&cta_clips, wsum);
  __syncthreads();
  if (threadIdx.x == 0 && cta_clips && p.clip) atomicAdd(p.clip, cta_clips);
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

__global__ void gelu_kernel(const uint16_t* __restrict__ x, uint16_t* __restrict__ y, int64_t n) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t nvec = n >> 3;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nvec; i += stride) {
    uint4 v = reinterpret_cast<const uint4*>(x)[i];
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) w[k] = gelu2_bits(w[k]);
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
                            int layout, bool gelu, cudaStream_t s) {
  QuantParams p;
  memcpy(&p.tab, &quant_table_for(sg), sizeof(QuantTable));
  p.x = x;
  p.codes = codes;
  p.scales = scales;
  p.clip = clip;
  p.M = M;
  p.K = K;
  p.ldx = ldx;
  p.inv6sg = (float)(1.0 / (6.0 * (double)sg));
  // Streaming units: kc = K if a row fits in a unit, else the largest divisor of
  // K that is a multiple of 64 (16 without the four-scale gather) and fits.
  {
    const int64_t gran = (K % 64 == 0) ? 64 : 16;
    int64_t kc = K;
    if (K > kQUnitElems) {
      kc = gran;
      for (int64_t c = (kQUnitElems / gran) * gran; c >= gran; c -= gran)
        if (K % c == 0) {
          kc = c;
          break;
        }
    }
    p.kc = kc;
    p.R = kQUnitElems / kc;
    p.col_units = K / kc;
    p.n_units = ((M + p.R - 1) / p.R) * p.col_units;
    p.nbu = (int)(kc / 16);
    p.step_rows = (32 * kQConsumerWarps) / p.nbu;
    p.step_blocks = (32 * kQConsumerWarps) % p.nbu;
    p.one_copy = (ldx == K && kc == K) ? 1 : 0;
  }
  // Exact clip threshold: smallest BF16 magnitude strictly beyond 2688 * s_g
  // (2688 * s_g is exact in FP64: 5 + 24 significant bits).
  p.clip_thr = clip_threshold_bits(sg);
  const bool tiled = layout == FH_SCALES_MMA_TILED;
  const bool gather4 = (K / 16) % 4 == 0;
  const int64_t want = p.n_units > 0 ? p.n_units : 1;
  const int grid = (int)(want < 2 * (int64_t)sm_count() ? want : 2 * (int64_t)sm_count());
  int dev = 0;
  cudaGetDevice(&dev);
  // Shared-memory opt-in of a kernel, once per device.
  auto configure = [&](auto kernel, DeviceTable& table) {
    const int v = per_device(table, dev, [&](int) {
      cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kQSmem);
      return e == cudaSuccess ? 1 : -(int)e;
    });
    return v > 0 ? cudaSuccess : (cudaError_t)(-v);
  };
  auto launch = [&](auto kernel, DeviceTable& table) {
    cudaError_t e = configure(kernel, table);
    if (e != cudaSuccess) return e;
    kernel<<<grid, kQThreads, kQSmem, s>>>(p);
    return cudaGetLastError();
  };
  static DeviceTable cfg_ft, cfg_ff, cfg_t[4];
  if (tiled) {
    // K % 64 == 0 here.  Units of 128 rows x 128 columns (two scale atoms)
    // when K allows, else 128 x 64.
    const int kg = (K % 128 == 0) ? 2 : 1;
    CUtensorMap tmx;
    if (!make_tensor_map_2d(&tmx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, (uint64_t)K, (uint64_t)M,
                            (uint64_t)ldx * 2, 64 * kg, 128, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorNotSupported;
    p.n_units = ((M + 127) / 128) * (K / (64 * kg));
    const int64_t tw = p.n_units > 0 ? p.n_units : 1;
    const int tgrid = (int)(tw < 2 * (int64_t)sm_count() ? tw : 2 * (int64_t)sm_count());
    auto kernel = kg == 2 ? (gelu ? quantize_tiled_kernel<true, 2> : quantize_tiled_kernel<false, 2>)
                          : (gelu ? quantize_tiled_kernel<true, 1> : quantize_tiled_kernel<false, 1>);
    cudaError_t e = configure(kernel, cfg_t[(gelu ? 1 : 0) + 2 * (kg - 1)]);
    if (e != cudaSuccess) return e;
    kernel<<<tgrid, kQThreads, kQSmem, s>>>(tmx, p);
    return cudaGetLastError();
  }
  return gather4 ? launch(quantize_kernel<true>, cfg_ft) : launch(quantize_kernel<false>, cfg_ff);
}

cudaError_t read_and_clear_quant_error(unsigned int* bits) {
  unsigned int v = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_quant_error, sizeof v);
  if (e != cudaSuccess) return e;
  e = cudaMemcpyToSymbol(g_quant_error, &zero, sizeof zero);
  *bits = v;
  return e;
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
