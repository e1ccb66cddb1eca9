// fh_int8.cu -- INT8 query/key quantization and INT8 attention scores on the
// sm_100a tensor cores.
//
// FastH3 Trim (comfyui-wiki news), "How fast it runs": the FP8 path of the
// RTX 4090 quantizes the query and the key to INT8 to compute the attention
// scores.  The pages fix neither the granularity nor the rounding; this file
// takes one symmetric scale per row (one token of one head):
//   s = fp32(amax_row / 127),  q = clamp(rne(fp32(x / s)), -127, 127)
// (IEEE single divisions; s = q = 0 for an all-zero row), and the scores
//   S[h, i, j] = ((float(acc) * (s_q[h, i] * sm_scale)) * s_k[h, j]),
//   acc = sum_d q[h, i, d] * k[h, j, d]   (exact, INT32 on the tensor cores).
//
// Score kernel: persistent, warp-specialized, one CTA per SM, 320 threads.
//   warp 0      TMA producer: per tile, the 128 query rows and 256 key rows
//               (128-byte rows, 128-byte swizzle) of one head, one 128-element
//               slice of d per stage; 3-D tensor maps (d, token, head) so that
//               rows past a head's token count, and columns past d, read as zero.
//   warp 1      allocates TMEM (two 256-column INT32 accumulators) and issues
//               tcgen05.mma kind::i8 (M = 128, N = 256, K = 32): four per stage.
//   warps 2..9  epilogue, two warps per TMEM lane quadrant (one per half of the
//               columns): pipelined tcgen05.ld, the FP32 scaling, a transpose
//               through shared memory and coalesced 16-byte stores (four whole
//               128-byte rows of S per instruction), while the MMA warp fills
//               the other accumulator.  S is write-bound: coalesced stores from
//               eight warps keep more of it in flight than per-SM TMA stores.
// No TMA load uses cluster multicast.  Every mbarrier wait is bounded; on
// expiry the kernel sets its error word and drains what it issued.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

#include "fh_internal.h"

namespace fh {

namespace {

__device__ unsigned int g_int8_error = 0;

// ---- row quantizer -------------------------------------------------------------

// The element decision shared by both row kernels: q = clamp(rne(x / s)).
__device__ __forceinline__ uint32_t int8_code(float xv, float s) {
  int qi = 0;
  if (s > 0.0f) qi = min(127, max(-127, __float2int_rn(__fdiv_rn(xv, s))));
  return (uint32_t)qi & 0xFFu;
}

// General form (any d % 8 == 0): one warp per row, two passes over the row.
__global__ void __launch_bounds__(256) int8_quantize_rows_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                                 int64_t d, int64_t ldx, int8_t* __restrict__ q,
                                                                 float* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    const uint16_t* xr = x + r * ldx;
    uint32_t mx = 0;  // max magnitude bits (BF16 magnitudes order like their bits)
    for (int64_t c = 8 * lane; c < d; c += 256) {
      const uint4 v = *reinterpret_cast<const uint4*>(xr + c);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) mx = max(mx, max(w[k] & 0x7FFFu, (w[k] >> 16) & 0x7FFFu));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
    const float s = __fdiv_rn(__uint_as_float(mx << 16), 127.0f);
    if (lane == 0) scales[r] = s;
    int8_t* qr = q + r * d;
    for (int64_t c = 8 * lane; c < d; c += 256) {
      const uint4 v = *reinterpret_cast<const uint4*>(xr + c);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t out[2] = {0, 0};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
#pragma unroll
        for (int hlf = 0; hlf < 2; ++hlf) {
          const float xv = __uint_as_float(hlf ? (w[k] & 0xFFFF0000u) : (w[k] << 16));
          out[k >> 1] |= int8_code(xv, s) << (8 * (2 * (k & 1) + hlf));
        }
      }
      *reinterpret_cast<uint2*>(qr + c) = make_uint2(out[0], out[1]);
    }
  }
}

// Register-resident form for d <= 2048: a group of G lanes holds RB rows of NC
// 16-byte chunks per lane, so each row is read from HBM once and the loads of
// RB rows are in flight together.  Chunks past d read as zero (they change no
// maximum) and are not stored.
template <int G, int NC, int RB>
__global__ void __launch_bounds__(256) int8_rows_reg_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t d,
                                                            int64_t ldx, int8_t* __restrict__ q,
                                                            float* __restrict__ scales) {
  static_assert(32 % G == 0 && NC >= 1 && RB >= 1, "group shape");
  const int lane = threadIdx.x & 31, sub = lane % G;
  constexpr int kGroupsPerBlock = 8 * (32 / G);
  const int64_t gid = (int64_t)blockIdx.x * kGroupsPerBlock + (threadIdx.x >> 5) * (32 / G) + lane / G;
  const int64_t stride = (int64_t)gridDim.x * kGroupsPerBlock * RB;
  // The loop runs on the warp's first group (rw), so that all 32 lanes take the
  // full-warp shuffles together; a group past the last row loads zeros and
  // stores nothing.
  for (int64_t r0 = gid * RB, rw = (gid - lane / G) * RB; rw < rows; r0 += stride, rw += stride) {
    uint4 v[RB][NC];
    uint32_t mx[RB];
#pragma unroll
    for (int b = 0; b < RB; ++b) {
#pragma unroll
      for (int i = 0; i < NC; ++i) {
        const int64_t c = (int64_t)(sub + G * i) * 8;
        v[b][i] = (r0 + b < rows && c < d) ? *reinterpret_cast<const uint4*>(x + (r0 + b) * ldx + c)
                                           : make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int b = 0; b < RB; ++b) {
      uint32_t m = 0;  // max magnitude bits (BF16 magnitudes order like their bits)
#pragma unroll
      for (int i = 0; i < NC; ++i) {
        const uint32_t w[4] = {v[b][i].x, v[b][i].y, v[b][i].z, v[b][i].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) m = max(m, max(w[k] & 0x7FFFu, (w[k] >> 16) & 0x7FFFu));
      }
#pragma unroll
      for (int o = G / 2; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
      mx[b] = m;
    }
#pragma unroll
    for (int b = 0; b < RB; ++b) {
      const int64_t r = r0 + b;
      if (r >= rows) break;
      const float sc = __fdiv_rn(__uint_as_float(mx[b] << 16), 127.0f);
      if (sub == 0) scales[r] = sc;
#pragma unroll
      for (int i = 0; i < NC; ++i) {
        const int64_t c = (int64_t)(sub + G * i) * 8;
        if (c >= d) break;
        const uint32_t w[4] = {v[b][i].x, v[b][i].y, v[b][i].z, v[b][i].w};
        uint32_t out[2] = {0, 0};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          out[k >> 1] |= int8_code(__uint_as_float(w[k] << 16), sc) << (16 * (k & 1));
          out[k >> 1] |= int8_code(__uint_as_float(w[k] & 0xFFFF0000u), sc) << (16 * (k & 1) + 8);
        }
        *reinterpret_cast<uint2*>(q + r * d + c) = make_uint2(out[0], out[1]);
      }
    }
  }
}

// ---- PTX helpers for the score kernel --------------------------------------------

__device__ __forceinline__ uint32_t s_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void bar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ bool bar_try_wait(uint32_t bar, uint32_t parity) {
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

__device__ __forceinline__ uint64_t now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait (~4 s, or until another role gave up): sets the error word and
// the CTA's abort flag on expiry.
__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t parity, volatile int* abort) {
  if (bar_try_wait(bar, parity)) return true;
  const uint64_t t0 = now_ns();
  for (uint32_t i = 1; i < (1u << 30); ++i) {
    if (bar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 0u) {
      if (*abort) return false;
      if (now_ns() - t0 > 4000000000ull) break;
    }
  }
  atomicOr(&g_int8_error, (unsigned)kDevErrTimeout);
  *abort = 1;
  return false;
}

// Drain wait: bounded by time only (~1 s), ignores the abort flag.
__device__ __forceinline__ void bar_drain(uint32_t bar, uint32_t parity) {
  if (bar_try_wait(bar, parity)) return;
  const uint64_t t0 = now_ns();
  for (uint32_t i = 1; i < (1u << 30); ++i) {
    if (bar_try_wait(bar, parity)) return;
    if ((i & 255u) == 0u && now_ns() - t0 > 1000000000ull) break;
  }
  atomicOr(&g_int8_error, (unsigned)kDevErrTimeout);
}

__device__ __forceinline__ bool elect() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "elect.sync _|p, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// K-major operand descriptor, 128-byte rows in 1024-byte swizzle atoms.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr) {
  uint64_t dsc = (uint64_t)((addr >> 4) & 0x3FFFu);
  dsc |= (uint64_t)1u << 16;
  dsc |= (uint64_t)(1024u >> 4) << 32;
  dsc |= (uint64_t)1u << 46;
  dsc |= (uint64_t)2u << 61;
  return dsc;
}

__device__ __forceinline__ void tmem_load_32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32"
      " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15,"
      " %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]),
        "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]),
        "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
}

// Completes the tcgen05.ld that wrote v; the registers are tied to the wait so
// that no use of them can be scheduled before it.
__device__ __forceinline__ void tmem_wait_32(uint32_t (&v)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]), "+r"(v[6]), "+r"(v[7]),
                 "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]), "+r"(v[12]), "+r"(v[13]), "+r"(v[14]),
                 "+r"(v[15]), "+r"(v[16]), "+r"(v[17]), "+r"(v[18]), "+r"(v[19]), "+r"(v[20]), "+r"(v[21]),
                 "+r"(v[22]), "+r"(v[23]), "+r"(v[24]), "+r"(v[25]), "+r"(v[26]), "+r"(v[27]), "+r"(v[28]),
                 "+r"(v[29]), "+r"(v[30]), "+r"(v[31])
               :
               : "memory");
}

// ---- score kernel ----------------------------------------------------------------

constexpr int kTM = 128;                  // query rows per tile
constexpr int kTN = 256;                  // key rows per tile
constexpr int kSK = 128;                  // d elements (bytes) per stage
constexpr int kMmaKI8 = 32;               // K of one tcgen05.mma kind::i8
constexpr int kStagesI8 = 2;
constexpr int kABytesI8 = kTM * kSK;      // 16384
constexpr int kBBytesI8 = kTN * kSK;      // 32768
constexpr int kEpiWarpsI8 = 8;                      // two per TMEM lane quadrant, one per column half
constexpr int kThreadsI8 = 32 * (2 + kEpiWarpsI8);  // 320
constexpr int kEpiCols = kTN / 2;                   // accumulator columns per epilogue warp
constexpr int kOutCols = 32;              // FP32 columns per epilogue chunk (128 bytes)
constexpr int kOutBufBytes = 32 * kOutCols * 4;     // 4096
constexpr int kOffAI8 = 0;
constexpr int kOffBI8 = kOffAI8 + kStagesI8 * kABytesI8;
constexpr int kOffOutI8 = kOffBI8 + kStagesI8 * kBBytesI8;
constexpr int kOffKsI8 = kOffOutI8 + kEpiWarpsI8 * kOutBufBytes;
constexpr int kOffBarI8 = kOffKsI8 + kEpiWarpsI8 * kEpiCols * 4;
constexpr int kNumBarsI8 = 2 * kStagesI8 + 4 + 1;  // full, empty; acc full (2), acc empty (2); drain
constexpr int kSmemI8 = kOffBarI8 + kNumBarsI8 * 8 + 16 + 1024;
// tcgen05.mma kind::i8: D S32 (bits 4-5 = 2), A and B signed 8-bit (1 at bits
// 7 and 10), both K-major, N >> 3 at bit 17, M >> 4 at bit 24.
constexpr uint32_t kIdescI8 = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kTN >> 3) << 17) |
                              ((uint32_t)(kTM >> 4) << 24);
static_assert(kSmemI8 <= 232448, "shared memory budget");
static_assert(kOffBI8 % 1024 == 0 && kOffOutI8 % 1024 == 0, "alignment");

struct ScoreParams {
  const float* q_scales;
  const float* k_scales;
  float* out;
  float sm_scale;
  int heads, tq, tk;
  int m_tiles, n_tiles, num_tiles, k_stages;
  int stall;  // test hook: CTA 0's MMA warp stops before its first MMA (0: off)
};

struct RingI8 {
  int slot = 0;
  uint32_t phase = 0;
  __device__ __forceinline__ void next(int n) {
    if (++slot == n) {
      slot = 0;
      phase ^= 1u;
    }
  }
};

// kAligned: Tk % 4 == 0, so the rows of S are 16-byte aligned and every store
// is a float4; otherwise element stores, each bounded.
template <bool kAligned>
__global__ void __launch_bounds__(kThreadsI8, 1)
    int8_scores_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const ScoreParams p) {
  constexpr int S = kStagesI8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = s_u32(smem);
  const uint32_t bar0 = sbase + kOffBarI8;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };
  auto accf_bar = [&](int a) { return bar0 + 8u * (2 * S + a); };
  auto acce_bar = [&](int a) { return bar0 + 8u * (2 * S + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * S + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffBarI8 + kNumBarsI8 * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffBarI8 + kNumBarsI8 * 8 + 8);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      bar_init(full_bar(s), 1);
      bar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      bar_init(accf_bar(a), 1);
      bar_init(acce_bar(a), kEpiWarpsI8);
    }
    bar_init(drain_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmQ)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmK)) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(s_u32(tmem_slot)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ===================== TMA producer =====================
    RingI8 st;
    bool ok = true;
    for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
      const int h = t / (p.m_tiles * p.n_tiles), rem = t % (p.m_tiles * p.n_tiles);
      const int m0 = (rem / p.n_tiles) * kTM, n0 = (rem % p.n_tiles) * kTN;
      for (int kt = 0; kt < p.k_stages; ++kt) {
        if (!__all_sync(0xFFFFFFFFu, bar_wait(empty_bar(st.slot), st.phase ^ 1u, abort_flag))) {
          ok = false;
          break;
        }
        if (elect()) {
          asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(full_bar(st.slot)),
                       "r"((uint32_t)(kABytesI8 + kBBytesI8))
                       : "memory");
          tma_load_3d(sbase + kOffAI8 + st.slot * kABytesI8, &tmQ, full_bar(st.slot), kt * kSK, m0, h);
          tma_load_3d(sbase + kOffBI8 + st.slot * kBBytesI8, &tmK, full_bar(st.slot), kt * kSK, n0, h);
        }
        __syncwarp();
        st.next(S);
      }
    }
    for (int s = 0; s < S; ++s) bar_drain(full_bar(s), (s < st.slot) ? st.phase : (st.phase ^ 1u));
  } else if (warp == 1) {
    // ===================== MMA issuer =====================
    RingI8 st;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    const uint64_t adesc0 = sw128_desc(sbase + kOffAI8);
    const uint64_t bdesc0 = sw128_desc(sbase + kOffBI8);
    for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
      if (!__all_sync(0xFFFFFFFFu, bar_wait(acce_bar(acc), acc_phase ^ 1u, abort_flag))) break;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kTN);
      for (int kt = 0; kt < p.k_stages; ++kt) {
        if (!__all_sync(0xFFFFFFFFu, bar_wait(full_bar(st.slot), st.phase, abort_flag))) {
          ok = false;
          break;
        }
        if (p.stall && blockIdx.x == 0) {
          // Test hook: stop without issuing or committing, so this CTA's
          // producer and epilogue run into their bounded waits.
          ok = false;
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint64_t adesc = adesc0 + (uint64_t)((st.slot * kABytesI8) >> 4);
        const uint64_t bdesc = bdesc0 + (uint64_t)((st.slot * kBBytesI8) >> 4);
        if (elect()) {
#pragma unroll
          for (int k = 0; k < kSK / kMmaKI8; ++k)
            asm volatile(
                "{\n\t.reg .pred p;\n\t"
                "setp.ne.b32 p, %4, 0;\n\t"
                "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
                "l"(adesc + (uint64_t)(k * kMmaKI8 / 16)), "l"(bdesc + (uint64_t)(k * kMmaKI8 / 16)),
                "r"(kIdescI8), "r"((kt | k) != 0 ? 1u : 0u)
                : "memory");
          asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                           empty_bar(st.slot))
                       : "memory");
        }
        __syncwarp();
        st.next(S);
      }
      if (!ok) break;
      if (elect())
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                         accf_bar(acc))
                     : "memory");
      __syncwarp();
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (elect())
      asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(drain_bar)
                   : "memory");
    __syncwarp();
    bar_drain(drain_bar, 0);
  } else {
    // ===================== epilogue =====================
    // Warp ew = warp - 2 reads TMEM lane quadrant warp % 4 (rows 32q .. 32q+31
    // of the tile) and accumulator columns [half * 128, half * 128 + 128).
    const int ew = warp - 2;
    const int q = warp & 3;
    const int col0 = (ew >> 2) * kEpiCols;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    uint8_t* out_buf = smem + kOffOutI8 + ew * kOutBufBytes;
    float* ks_s = reinterpret_cast<float*>(smem + kOffKsI8) + ew * kEpiCols;
    int acc = 0;
    uint32_t acc_phase = 0;
    // The scales of a tile are loaded into registers one tile ahead, so that
    // their global-load latency overlaps the previous tile's epilogue.
    constexpr int kKsPerLane = kEpiCols / 32;
    float ks_next[kKsPerLane], qs_next = 0.0f;
    auto load_scales = [&](int t) {
      const int h = t / (p.m_tiles * p.n_tiles), rem = t % (p.m_tiles * p.n_tiles);
      const int m0 = (rem / p.n_tiles) * kTM, n0 = (rem % p.n_tiles) * kTN + col0;
      const int row = m0 + 32 * q + lane;
#pragma unroll
      for (int i = 0; i < kKsPerLane; ++i) {
        const int col = n0 + lane + 32 * i;
        ks_next[i] = (col < p.tk) ? p.k_scales[(size_t)h * p.tk + col] : 0.0f;
      }
      qs_next = (row < p.tq) ? p.q_scales[(size_t)h * p.tq + row] : 0.0f;
    };
    if (blockIdx.x < p.num_tiles) load_scales(blockIdx.x);
    for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x) {
      const int h = t / (p.m_tiles * p.n_tiles), rem = t % (p.m_tiles * p.n_tiles);
      const int m0 = (rem / p.n_tiles) * kTM, n0 = (rem % p.n_tiles) * kTN + col0;
      // This warp's copy of its columns' key scales (4 per lane).
#pragma unroll
      for (int i = 0; i < kKsPerLane; ++i) ks_s[lane + 32 * i] = ks_next[i];
      const float qs = qs_next * p.sm_scale;
      __syncwarp();
      if (t + (int)gridDim.x < p.num_tiles) load_scales(t + gridDim.x);
      if (!__all_sync(0xFFFFFFFFu, bar_wait(accf_bar(acc), acc_phase, abort_flag))) break;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t tcol = tmem_base + lane_base + (uint32_t)(acc * kTN + col0);
      // Chunk c's TMEM load is in flight while chunk c - 1 is scaled and stored.
      uint32_t va[32], vb[32];
      tmem_load_32(tcol, va);
      tmem_wait_32(va);
      auto emit = [&](const uint32_t(&v)[32], int c) {
        float o[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) o[j] = ((float)(int32_t)v[j] * qs) * ks_s[c * kOutCols + j];
        // Transpose through a 128-byte-swizzled staging buffer (thread = row on
        // the way in, eight lanes per row on the way out), so that every store
        // instruction writes four whole 128-byte rows of S.
        uint8_t* sb = out_buf;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t chunk = (uint32_t)i ^ ((uint32_t)lane & 7u);
          *reinterpret_cast<float4*>(sb + lane * 128 + chunk * 16) =
              make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
        }
        __syncwarp();
        const int gcol = n0 + c * kOutCols + 4 * (lane & 7);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = 4 * i + (lane >> 3);
          const float4 val =
              *reinterpret_cast<const float4*>(sb + r * 128 + (((uint32_t)(lane & 7) ^ (uint32_t)(r & 7)) * 16));
          const int grow = m0 + 32 * q + r;
          if constexpr (kAligned) {  // a float4 never straddles tk
            if (grow < p.tq && gcol < p.tk)
              *reinterpret_cast<float4*>(p.out + ((size_t)h * p.tq + grow) * p.tk + gcol) = val;
          } else {
            if (grow < p.tq) {
              float* dst = p.out + ((size_t)h * p.tq + grow) * p.tk + gcol;
              if (gcol < p.tk) dst[0] = val.x;
              if (gcol + 1 < p.tk) dst[1] = val.y;
              if (gcol + 2 < p.tk) dst[2] = val.z;
              if (gcol + 3 < p.tk) dst[3] = val.w;
            }
          }
        }
        __syncwarp();  // the buffer is rewritten by the next chunk
      };
      static_assert(kEpiCols / kOutCols == 4, "the pipelined epilogue below handles four chunks");
      tmem_load_32(tcol + 32, vb);
      emit(va, 0);
      tmem_wait_32(vb);
      tmem_load_32(tcol + 64, va);
      emit(vb, 1);
      tmem_wait_32(va);
      tmem_load_32(tcol + 96, vb);
      emit(va, 2);
      tmem_wait_32(vb);
      // Every TMEM read of this accumulator is complete: release it to the MMA.
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(acce_bar(acc)) : "memory");
      emit(vb, 3);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  if (warp == 1) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(512));
  }
}

// ---- host ----------------------------------------------------------------------

typedef CUresult (*EncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                             const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                             CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode3() {
  // Looked up once per process (thread-safe static initialization).
  static const EncodeFn fn = []() -> EncodeFn {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeFn>(ptr);
    return nullptr;
  }();
  return fn;
}

// 3-D map of a [heads][rows][inner] array with a box of box_inner x box_rows x 1.
bool map3(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t rows, uint64_t heads,
          uint64_t elem_bytes, uint32_t box_inner, uint32_t box_rows) {
  EncodeFn fn = encode3();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {inner, rows, heads};
  const cuuint64_t strides[2] = {inner * elem_bytes, inner * rows * elem_bytes};
  const cuuint32_t box[3] = {box_inner, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_int8_quantize_rows(const uint16_t* x, int64_t rows, int64_t d, int64_t ldx, int8_t* q,
                                      float* scales, cudaStream_t s) {
  // Rows per block of each form; the grid covers the rows once, up to 8 blocks
  // of 256 threads per SM, with a grid-stride loop beyond that.
  const int64_t cap = (int64_t)sm_count() * 8;
  auto grid_for = [&](int64_t rows_per_block) {
    const int64_t need = (rows + rows_per_block - 1) / rows_per_block;
    return (int)(need < cap ? (need > 0 ? need : 1) : cap);
  };
  const int64_t chunks = d / 8;  // 16-byte chunks per row
  if (chunks <= 4)
    int8_rows_reg_kernel<4, 1, 2><<<grid_for(8 * 8 * 2), 256, 0, s>>>(x, rows, d, ldx, q, scales);
  else if (chunks <= 8)
    int8_rows_reg_kernel<8, 1, 2><<<grid_for(8 * 4 * 2), 256, 0, s>>>(x, rows, d, ldx, q, scales);
  else if (chunks <= 16)
    int8_rows_reg_kernel<16, 1, 2><<<grid_for(8 * 2 * 2), 256, 0, s>>>(x, rows, d, ldx, q, scales);
  else if (chunks <= 32)
    int8_rows_reg_kernel<32, 1, 2><<<grid_for(8 * 2), 256, 0, s>>>(x, rows, d, ldx, q, scales);
  else if (chunks <= 64)
    int8_rows_reg_kernel<32, 2, 2><<<grid_for(8 * 2), 256, 0, s>>>(x, rows, d, ldx, q, scales);
  else if (chunks <= 128)
    int8_rows_reg_kernel<32, 4, 1><<<grid_for(8), 256, 0, s>>>(x, rows, d, ldx, q, scales);
  else if (chunks <= 256)
    int8_rows_reg_kernel<32, 8, 1><<<grid_for(8), 256, 0, s>>>(x, rows, d, ldx, q, scales);
  else
    int8_quantize_rows_kernel<<<grid_for(8), 256, 0, s>>>(x, rows, d, ldx, q, scales);
  return cudaGetLastError();
}

cudaError_t launch_int8_scores(const int8_t* q, const float* q_scales, const int8_t* k, const float* k_scales,
                               float sm_scale, float* out, int64_t heads, int64_t tq, int64_t tk, int64_t d,
                               cudaStream_t s, const char** why) {
  CUtensorMap tmQ, tmK;
  if (!map3(&tmQ, CU_TENSOR_MAP_DATA_TYPE_UINT8, q, (uint64_t)d, (uint64_t)tq, (uint64_t)heads, 1, kSK, kTM) ||
      !map3(&tmK, CU_TENSOR_MAP_DATA_TYPE_UINT8, k, (uint64_t)d, (uint64_t)tk, (uint64_t)heads, 1, kSK, kTN)) {
    *why = "cuTensorMapEncodeTiled failed (driver entry point missing or a layout rule violated)";
    return cudaErrorNotSupported;
  }
  ScoreParams p;
  p.q_scales = q_scales;
  p.k_scales = k_scales;
  p.out = out;
  p.sm_scale = sm_scale;
  p.heads = (int)heads;
  p.tq = (int)tq;
  p.tk = (int)tk;
  p.m_tiles = (int)((tq + kTM - 1) / kTM);
  p.n_tiles = (int)((tk + kTN - 1) / kTN);
  p.num_tiles = (int)heads * p.m_tiles * p.n_tiles;
  p.k_stages = (int)((d + kSK - 1) / kSK);  // the last stage's columns past d read as zero
  const char* stall_env = getenv("FH_INT8_TEST_STALL");  // read at each launch
  p.stall = (stall_env != nullptr && stall_env[0] == '1') ? 1 : 0;
  static DeviceTable configured;
  int dev = 0;
  cudaGetDevice(&dev);
  const int cfg = per_device(configured, dev, [](int) {
    cudaError_t e = cudaFuncSetAttribute(int8_scores_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemI8);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(int8_scores_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemI8);
    return e == cudaSuccess ? 1 : -(int)e;
  });
  if (cfg <= 0) return (cudaError_t)(-cfg);
  const int grid = p.num_tiles < sm_count() ? p.num_tiles : sm_count();
  if (tk % 4 == 0)
    int8_scores_kernel<true><<<grid, kThreadsI8, kSmemI8, s>>>(tmQ, tmK, p);
  else
    int8_scores_kernel<false><<<grid, kThreadsI8, kSmemI8, s>>>(tmQ, tmK, p);
  return cudaGetLastError();
}

cudaError_t read_and_clear_int8_error(unsigned int* bits) {
  unsigned int v = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_int8_error, sizeof v);
  if (e != cudaSuccess) return e;
  e = cudaMemcpyToSymbol(g_int8_error, &zero, sizeof zero);
  *bits = v;
  return e;
}

}  // namespace fh
