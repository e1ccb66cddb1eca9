// fh_gemm.cu -- NVFP4 linear layer on the sm_100a tcgen05 tensor cores.
//
//   y[m, n] = bf16( alpha * sum_k A[m,k] W[n,k] + bias[n] ),  alpha = s_gA * s_gW
//
// with A, W NVFP4 (E2M1 codes, one E4M3 scale per 16 elements along K).  This
// is the FP4 matmul that FastH3 runs on Blackwell tensor cores (FastH3 thread
// digest, farwalk.ai, tweet 5/8; FastH3 Trim, comfyui-wiki news, "How fast it
// runs": the RTX 4090 lacks FP4 tensor cores, Blackwell has them).
//
// Design: persistent, warp-specialized, one CTA per SM.  By default two CTAs
// of a cluster pair up on one 256 x 256 output tile with tcgen05.mma
// cta_group::2 (each SM computes 128 rows; the 256 W rows are split 128/128
// between the two SMs' shared memory, so each SM loads and holds half of W);
// the single-CTA form (128 x 192 tiles) is the same code with kCta = 1.
// Two tile forms (template parameter BN):
//   256 (default, CTA pair): 256 x 256 output tiles, one 256-column TMEM
//       accumulator per CTA, 5 stages, 320 threads;
//   192 (CTA pair, or single CTA): 256 x 192 (128 x 192) tiles, two 192-column
//       accumulators, 6 (4) stages, 192 threads.
// Roles per CTA:
//   warp 0      TMA producer: per 256-wide K stage, its 128 x 128-byte A tile,
//               its (BN / kCta) x 128-byte W tile (128-byte swizzle), and the
//               stage's scale atoms (512 bytes = 128 rows x 64 K; one box for
//               this CTA's A rows, one for the tile's two W scale blocks), all
//               by tensor TMA completing on the leader CTA's stage barrier.
//   warp 1      allocates TMEM (512 columns, both CTAs); in the leader CTA one
//               lane copies the stage's scale atoms from shared memory into one
//               of two TMEM scale buffers (tcgen05.cp 32x128b.warpx4, which
//               replicates each atom into the four lane quadrants, in both CTAs
//               of the pair) and then issues four tcgen05.mma kind::mxf4nvf4
//               block_scale (M = 128 kCta, N = BN, K = 64) into an accumulator.
//               Copies and MMAs run in issue order on the tensor pipe, so a
//               scale buffer needs no barrier; double buffering keeps a copy
//               from waiting on the MMAs still reading the other.
//               tcgen05.commit (multicast to the pair) frees the stage's shared
//               memory and, after the last stage, hands the accumulator to both
//               CTAs' epilogues.
//   warps 2..   epilogue (4 warps for BN = 192, one per TMEM lane quadrant; 8
//               for BN = 256, two per quadrant, one per 128-column half):
//               tcgen05.ld of their TMEM lanes, alpha * acc + bias in FP32,
//               BF16 round-to-nearest-even, 128-byte-swizzled staging in shared
//               memory and TMA stores.  With two accumulators this overlaps the
//               MMAs of the next tile; with one, each warp first copies its 128
//               columns into registers and releases the accumulator, so the
//               MMAs wait only for that copy.
// TMEM columns (each CTA): the accumulators from 0, then two scale buffers of
// 48 columns: per K=64 step, 4 columns of A scales (row r at lane r%32, column
// r/32) then 8 columns of W scales (the two 128-row scale blocks the tile's
// rows fall in; a 192-row tile reads 6 of them from column 0 or 2).
// No TMA load uses cluster multicast; only tcgen05.commit is multicast.
// Every mbarrier wait is bounded; on expiry the kernel sets the device error
// word, stops issuing work, drains what it issued and frees its TMEM.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "fh_internal.h"

namespace fh {

namespace {

__device__ unsigned int g_device_error = 0;

constexpr int BK = 256;                  // FP4 elements per stage = 128 bytes per row
constexpr int kMmaK = 64;                // K of one tcgen05.mma kind::mxf4nvf4
constexpr int kKSteps = BK / kMmaK;      // 4
constexpr int kAtomBytes = 512;          // 128 rows x 4 scales
constexpr int kABytes = 128 * BK / 2;    // 16384: one CTA's 128 A rows
constexpr int kSFABytes = kKSteps * kAtomBytes;      // 2048
constexpr int kSFBBytes = 2 * kKSteps * kAtomBytes;  // 4096
constexpr int kEpiCols = 64;                          // columns per TMA store box
constexpr int kEpiBufBytes = 32 * kEpiCols * 2;       // 4096: 32 rows x 128 bytes
constexpr int kTmemCols = 512;
constexpr int kSfCols = 4 * kKSteps + 8 * kKSteps;    // 48 per stage: A 4, W 8 per K=64 step
constexpr int kSfBufs = 2;

// Two tile forms share the kernel.  BN = 192: two 192-column accumulators, so
// an epilogue overlaps the next tile's MMAs entirely; four epilogue warps.
// BN = 256 (CTA pair only): one 256-column accumulator -- two would fill TMEM
// -- drained into registers by eight epilogue warps (two per TMEM lane
// quadrant, one per 128-column half), which release it before they scale,
// round and store; each stage then feeds 33% more MACs from 12% more bytes.
// kPro = 1 (256-wide pair form only): the activations arrive in BF16 and two
// more warps per CTA quantize them inside the kernel (see the prologue
// quantizer below); one stage fewer makes room for their decision table.
template <int kCta, int kBN, int kPro = 0>
struct Cfg {
  static_assert(kBN == 192 || (kBN == 256 && kCta == 2), "tile forms");
  static_assert(kPro == 0 || (kBN == 256 && kCta == 2), "the quantizing prologue runs in the 256-wide pair form");
  static constexpr int BN = kBN;                       // output columns per tile
  static constexpr int BM = 128 * kCta;                // output rows per tile
  static constexpr int kBRows = BN / kCta;             // W rows each CTA loads
  static constexpr int kAccBufs = BN == 256 ? 1 : 2;   // TMEM accumulators
  static constexpr int kEpiWarps = BN == 256 ? 8 : 4;
  static constexpr int kWarpCols = BN == 256 ? 128 : BN;  // accumulator columns per epilogue warp
  static constexpr int kQuantWarps = kPro ? 2 : 0;     // prologue quantizer warps (warps 2, 3)
  static constexpr int kEpiWarp0 = 2 + kQuantWarps;    // first epilogue warp
  static constexpr int kThreads = 64 + 32 * kQuantWarps + 32 * kEpiWarps;
  static constexpr int kSfCol0 = kAccBufs * BN;        // first TMEM column of the scale buffers
  static constexpr int kStages = BN == 256 ? (kPro ? 4 : 5) : (kCta == 2 ? 6 : 4);
  static constexpr int kEpiBufs = kCta == 2 ? 1 : 2;   // output staging buffers per epilogue warp
  static constexpr int kBBytes = kBRows * BK / 2;
  static constexpr int kOffA = 0;
  static constexpr int kOffB = kOffA + kStages * kABytes;
  static constexpr int kOffSFA = kOffB + kStages * kBBytes;
  static constexpr int kOffSFB = kOffSFA + kStages * kSFABytes;
  static constexpr int kOffEpi = kOffSFB + kStages * kSFBBytes;
  static constexpr int kOffBias = kOffEpi + kEpiWarps * kEpiBufs * kEpiBufBytes;
  static constexpr int kOffQTab = kOffBias + kEpiWarps * kWarpCols * 2;  // prologue decision table
  static constexpr int kOffBar = kOffQTab + (kPro ? (int)sizeof(QuantTable) : 0);
  // full, empty (per stage); acc full, acc empty (per accumulator); drain;
  // the peer producer's end-of-loading report (leader CTA)
  static constexpr int kNumBars = 2 * kStages + 2 * kAccBufs + 2;
  static constexpr int kSmemBytes = kOffBar + kNumBars * 8 + 16;
  static constexpr int kSmemAlloc = kSmemBytes + 1024;  // slack for 1024-byte alignment
  // Instruction descriptor of tcgen05.mma kind::mxf4nvf4: A and B E2M1
  // (format 1), both K-major, UE4M3 scales, N >> 3 at bit 17, M >> 4 at bit
  // 24, dense, K = 64, scale-factor ids 0.
  static constexpr uint32_t kIdesc =
      (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
  static_assert(kOffB % 1024 == 0 && kOffSFA % 1024 == 0 && kOffEpi % 1024 == 0, "alignment");
  static_assert(kBBytes % 1024 == 0, "W stage alignment");
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
  static_assert(kSfCol0 + kSfBufs * kSfCols <= kTmemCols, "TMEM budget");
};

struct Params {
  const uint16_t* bias;
  float alpha;
  int M, N, K;
  int n_tiles, num_tiles, k_stages;
  int ksteps_total;  // K / 64
  int stall_group;   // test hook: CTA group that stalls (-1: none) ...
  int stall_mode;    // ... 1: its MMA warp stops after 3 stages; 2: its second CTA's producer stops after 2
};

// Epilogue mode 1: instead of y, emit the next layer's NVFP4 input
// g = GELU(bf16(alpha * acc + bias)) quantized with that layer's global scale:
// codes [M, N/2] and tensor-core-layout scales of [M, N] (N % 64 == 0), plus
// the count of clipped elements of g.
struct EpiQuant {
  QuantTable tab;  // decision table of the next layer's global scale
  uint8_t* codes;
  uint8_t* scales;
  unsigned long long* clip;  // may be null
  float inv6sg;
  uint32_t clip_thr;
  int katoms;  // N / 64: scale atoms per 128-row block
  int m_pad;   // rows of the scale array: ceil(M / 128) * 128
};
struct EpiNone {};
template <int kEpi>
struct EpiSel {
  using type = EpiNone;
};
template <>
struct EpiSel<1> {
  using type = EpiQuant;
};

// Prologue mode 1: the activations x [M, K] arrive in BF16 and the kernel
// quantizes them itself.  Two warps of every CTA walk the quantization items
// (32 rows x 64 columns each) in row-block order and write the codes and
// tensor-core-layout scales to global memory (outputs the caller owns; they
// stay in L2 for the tiles that read them), then count the item in the row
// block's ready counter.  A producer loads a row block's A tiles only once
// its counter has seen all 4 * K/64 items.  All CTAs of the grid are resident
// at once (the grid is sized to the clusters that fit), so every item a
// producer waits for is being worked on.  The counters start at zero; the
// last CTA to leave sets them back to zero.
struct ProQuant {
  QuantTable tab;     // decision table of the activations' global scale
  const uint16_t* x;  // BF16 [M, K], rows ldx elements apart
  uint8_t* codes;     // [M, K/2]
  uint8_t* scales;    // tensor-core layout of [M, K]
  unsigned long long* clip;  // may be null
  uint32_t* sync;     // n_rb ready counters, then the exit counter
  int64_t ldx;
  float inv6sg;
  uint32_t clip_thr;
  int katoms;  // K / 64
  int n_rb;    // ceil(M / 128)
};
struct ProNone {};
template <int kPro>
struct ProSel {
  using type = ProNone;
};
template <>
struct ProSel<1> {
  using type = ProQuant;
};


__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}


__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
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

// One lane of the (converged) warp; the whole warp runs the issuing loops so
// that every operand of the tcgen05 / TMA instructions stays warp-uniform.
__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "elect.sync _|p, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait for phase `parity` of an mbarrier.  Gives up after ~4 s (or
// when another role of the CTA already gave up), setting the device error word
// and the CTA's abort flag.
constexpr uint64_t kWaitLimitNs = 4000000000ull;
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort,
                                             uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t i = 1; i < (1u << 30); ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 0u) {
      if (*abort) return false;
      if (global_ns() - t0 > limit_ns) break;
    }
  }
  atomicOr(&g_device_error, (unsigned)kDevErrTimeout);
  *abort = 1;
  return false;
}

// Wait used while draining before exit: copies and MMAs this CTA issued must
// have completed before it frees TMEM or retires, so this wait ignores the
// abort flag and gives up only on its own time limit (~1 s).
constexpr uint64_t kDrainLimitNs = 1000000000ull;
__device__ __forceinline__ void wait_drain(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = global_ns();
  for (uint32_t i = 1; i < (1u << 30); ++i) {
    if (mbar_try_wait(bar, parity)) return;
    if ((i & 255u) == 0u && global_ns() - t0 > kDrainLimitNs) break;
  }
  atomicOr(&g_device_error, (unsigned)kDevErrTimeout);
}

// Wait for the peer producer's end-of-loading report (an arrival with release
// semantics at cluster scope).  The peer reports once its own waits have
// ended, which can take one full wait limit after this CTA stopped, so this
// waits for the wait limit plus the drain limit before giving up.
__device__ __forceinline__ bool wait_report(uint32_t bar) {
  const uint64_t t0 = global_ns();
  for (uint32_t i = 0; i < (1u << 30); ++i) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], 0;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar)
        : "memory");
    if (ok) return true;
    if ((i & 255u) == 0u && global_ns() - t0 > kWaitLimitNs + kDrainLimitNs) break;
  }
  atomicOr(&g_device_error, (unsigned)kDevErrTimeout);
  return false;
}

// Tensor TMA load into this CTA's shared memory.  kCta == 2: `bar` may be the
// leader CTA's barrier (a shared::cluster address); no multicast.
template <int kCta>
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y) {
  if (kCta == 1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
        : "memory");
  } else {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
        : "memory");
  }
}

// Address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}

// Arrive on a barrier given by its shared::cluster address (possibly in the
// peer CTA).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx_cluster(uint32_t cluster_bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cluster.b64 _, [%0], %1;" ::"r"(cluster_bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// The leader CTA's copy of a barrier of this CTA: its shared::cluster address
// for a pair, the barrier itself for a single CTA.
template <int kCta>
__device__ __forceinline__ uint32_t leader_bar(uint32_t local) {
  return kCta == 2 ? map_to_rank(local, 0) : local;
}

template <int kCta>
__device__ __forceinline__ void arrive_leader(uint32_t bar) {
  if (kCta == 2)
    mbar_arrive_cluster(bar);
  else
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

template <int kCta>
__device__ __forceinline__ void arrive_expect_tx_leader(uint32_t bar, uint32_t bytes) {
  if (kCta == 2)
    mbar_arrive_expect_tx_cluster(bar, bytes);
  else
    mbar_arrive_expect_tx(bar, bytes);
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(x), "r"(y)
               : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read_1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrive on `bar` (in this CTA, or at the same offset in every CTA of the
// pair) once every tcgen05 operation this thread issued has completed.
template <int kCta>
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  if (kCta == 1) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
  } else {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            bar),
        "h"((uint16_t)3)
        : "memory");
  }
}

__device__ __forceinline__ void tc_commit_local2(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// Shared-memory matrix descriptor, K-major.  swizzle128: 128-byte rows in
// 1024-byte swizzle atoms (stride between 8-row groups 1024 bytes); otherwise
// no swizzle with 16-byte rows (stride between 8-row groups 128 bytes).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, bool swizzle128) {
  uint64_t d = (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;                            // leading byte offset (unused here)
  d |= (uint64_t)((swizzle128 ? 1024u : 128u) >> 4) << 32;  // stride byte offset
  d |= (uint64_t)1u << 46;                            // descriptor version (sm_100)
  d |= (uint64_t)(swizzle128 ? 2u : 0u) << 61;        // layout type
  return d;
}

template <int kCta>
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate, uint32_t sfa_tmem, uint32_t sfb_tmem) {
  if (kCta == 1) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X"
        " [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X"
        " [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
  }
}

// Copy one 512-byte scale atom (32 rows of 16 bytes: rows r, r+32, r+64, r+96
// at row r) into four TMEM columns, replicated into all four lane quadrants --
// the layout the block-scaled MMA reads.  kCta == 2: in both CTAs of the pair,
// each from its own shared memory at the same offset.
template <int kCta>
__device__ __forceinline__ void tc_cp_atom(uint32_t taddr, uint64_t sdesc) {
  if (kCta == 1)
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
  else
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// 32 consecutive TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld_32(uint32_t taddr, uint32_t (&v)[32]) {
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

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Registers written by tcgen05.ld are valid only after the wait; tying them to
// an asm statement placed after it keeps every use of them below the wait.
__device__ __forceinline__ void tie32(uint32_t* v) {
  asm volatile(""
               : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]), "+r"(v[6]), "+r"(v[7]),
                 "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]), "+r"(v[12]), "+r"(v[13]), "+r"(v[14]),
                 "+r"(v[15]), "+r"(v[16]), "+r"(v[17]), "+r"(v[18]), "+r"(v[19]), "+r"(v[20]), "+r"(v[21]),
                 "+r"(v[22]), "+r"(v[23]), "+r"(v[24]), "+r"(v[25]), "+r"(v[26]), "+r"(v[27]), "+r"(v[28]),
                 "+r"(v[29]), "+r"(v[30]), "+r"(v[31]));
}

template <int kC>
__device__ __forceinline__ void tmem_ld_wait_tied(uint32_t (&v)[kC][64]) {
  tmem_ld_wait();
#pragma unroll
  for (int c = 0; c < kC; ++c) {
    tie32(&v[c][0]);
    tie32(&v[c][32]);
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// ---- kernel ----------------------------------------------------------------

// Phase bookkeeping of a ring of `n` mbarrier-guarded slots.
struct Ring {
  int slot = 0;
  uint32_t phase = 0;
  __device__ __forceinline__ void next(int n) {
    if (++slot == n) {
      slot = 0;
      phase ^= 1u;
    }
  }
};

// ---- prologue quantizer (kPro = 1) ----------------------------------------------

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.global.acquire.gpu.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Bounded wait (about 4 s) until the counter reaches `target`; the whole warp
// polls the same word.  The async proxy (the tensor copies that follow) then
// sees what the counted items wrote.
__device__ __forceinline__ bool wait_counter(const uint32_t* ctr, uint32_t target, volatile int* abort) {
  const uint64_t t0 = global_ns();
  for (uint32_t i = 0; i < (1u << 30); ++i) {
    if (ld_acquire_u32(ctr) >= target) {
      asm volatile("fence.proxy.async.global;" ::: "memory");
      return true;
    }
    if (*abort) return false;
    if ((i & 15u) == 15u && global_ns() - t0 > kWaitLimitNs) break;
    __nanosleep(64);
  }
  atomicOr(&g_device_error, (unsigned)kDevErrTimeout);
  *abort = 1;
  return false;
}

// One quantization item: rows rb*128 + r1*32 .. +31, columns kc*64 .. +63 of
// x.  Lane l holds rows r1*32 + (l >> 2) + 8 i (i = 0..3), block l & 3.
struct ProItem {
  uint32_t w[4][8];
};

__device__ __forceinline__ void pro_item_coords(const ProQuant& pq, int item, int& rb, int& r1, int& kc) {
  const int per_rb = 4 * pq.katoms;
  rb = item / per_rb;
  const int rest = item - rb * per_rb;
  r1 = rest / pq.katoms;
  kc = rest - r1 * pq.katoms;
}

__device__ __forceinline__ void pro_load(const ProQuant& pq, int M, int item, int lane, ProItem& it) {
  int rb, r1, kc;
  pro_item_coords(pq, item, rb, r1, kc);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int row = rb * 128 + r1 * 32 + (lane >> 2) + 8 * i;
    uint4 a = make_uint4(0, 0, 0, 0), b = make_uint4(0, 0, 0, 0);
    if (row < M) {
      const uint4* src = reinterpret_cast<const uint4*>(pq.x + (int64_t)row * pq.ldx + kc * 64 + (lane & 3) * 16);
      a = __ldcs(src);
      b = __ldcs(src + 1);
    }
    it.w[i][0] = a.x; it.w[i][1] = a.y; it.w[i][2] = a.z; it.w[i][3] = a.w;
    it.w[i][4] = b.x; it.w[i][5] = b.y; it.w[i][6] = b.z; it.w[i][7] = b.w;
  }
}

__device__ __forceinline__ void pro_quantize_store(const ProQuant& pq, const QuantTable& tab, int M, int K, int item,
                                                   int lane, ProItem& it, unsigned long long& clips) {
  int rb, r1, kc;
  pro_item_coords(pq, item, rb, r1, kc);
  const int j = lane & 3;
  uint8_t* atom = pq.scales + ((size_t)rb * pq.katoms + kc) * 512;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r0 = (lane >> 2) + 8 * i;
    const int row = rb * 128 + r1 * 32 + r0;
    uint32_t amax;
    uint2 cd;
    uint32_t sc = nvfp4::quantize_block_codes(tab, pq.inv6sg, it.w[i], amax, cd);
    if (row < M) {
      *reinterpret_cast<uint2*>(pq.codes + (size_t)row * (size_t)(K >> 1) + kc * 32 + j * 8) = cd;
      clips += nvfp4::block_clips(it.w[i], amax, pq.clip_thr);
    } else {
      sc = 0;  // padding rows of the scale layout hold zero scales
    }
    const uint32_t pair = sc | (__shfl_down_sync(0xFFFFFFFFu, sc, 1) << 8);
    const uint32_t word = pair | (__shfl_down_sync(0xFFFFFFFFu, pair, 2) << 16);
    if (j == 0) *reinterpret_cast<uint32_t*>(atom + r0 * 16 + r1 * 4) = word;
  }
}

// Items are taken in chunks of kProChunk consecutive items of one row block
// (4 * K/64 items per row block, so a chunk never straddles two): within a
// chunk the next item's loads are in flight while the current one is
// quantized, and the chunk is published with one fence and one count.
constexpr int kProChunk = 4;

// Publish a chunk: every lane's stores, then kProChunk counts in the row
// block's counter (release), visible to the tensor copies of any CTA.
__device__ __forceinline__ void pro_publish(const ProQuant& pq, int rb, int lane) {
  asm volatile("fence.proxy.async.global;" ::: "memory");
  __threadfence();
  __syncwarp();
  if (lane == 0) atomicAdd(pq.sync + rb, (uint32_t)kProChunk);
}

template <int kCta, int kEpi, int kBN, int kPro>
__global__ void __launch_bounds__(Cfg<kCta, kBN, kPro>::kThreads, 1)
    nvfp4_linear_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
                        const __grid_constant__ CUtensorMap tmY, const Params p,
                        const __grid_constant__ typename EpiSel<kEpi>::type eq,
                        const __grid_constant__ typename ProSel<kPro>::type pq) {
  using C = Cfg<kCta, kBN, kPro>;
  constexpr int S = C::kStages;
  constexpr int BN = C::BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::kOffBar;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };            // leader: A, W and scales landed (both CTAs)
  auto empty_bar = [&](int s) { return bar0 + 8u * (S + s); };     // each CTA: stage free again
  auto accf_bar = [&](int a) { return bar0 + 8u * (2 * S + a); };  // each CTA: accumulator ready
  auto acce_bar = [&](int a) { return bar0 + 8u * (2 * S + C::kAccBufs + a); };  // leader: accumulator drained
  const uint32_t drain_bar = bar0 + 8u * (2 * S + 2 * C::kAccBufs);
  const uint32_t report_bar = drain_bar + 8u;  // leader: the peer producer reported its stage count
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffBar + C::kNumBars * 8);
  volatile uint32_t* peer_issued = reinterpret_cast<volatile uint32_t*>(smem + C::kOffBar + C::kNumBars * 8 + 12);
  if constexpr (kEpi == 1) {
    // The next layer's decision table, in the (otherwise unused) output staging area.
    static_assert(sizeof(QuantTable) <= C::kEpiWarps * C::kEpiBufs * kEpiBufBytes, "table fits the staging area");
    const uint4* src = reinterpret_cast<const uint4*>(&eq.tab);
    uint4* dst = reinterpret_cast<uint4*>(smem + C::kOffEpi);
    for (int i = threadIdx.x; i < (int)(sizeof(QuantTable) / 16); i += blockDim.x) dst[i] = src[i];
  }
  if constexpr (kPro == 1) {
    const uint4* src = reinterpret_cast<const uint4*>(&pq.tab);
    uint4* dst = reinterpret_cast<uint4*>(smem + C::kOffQTab);
    for (int i = threadIdx.x; i < (int)(sizeof(QuantTable) / 16); i += blockDim.x) dst[i] = src[i];
  }
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffBar + C::kNumBars * 8 + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = kCta == 2 ? cluster_rank() : 0u;
  const bool leader = rank == 0;
  const int pair = kCta == 2 ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int npairs = kCta == 2 ? (int)(gridDim.x >> 1) : (int)gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), kCta);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < C::kAccBufs; ++a) {
      mbar_init(accf_bar(a), 1);
      mbar_init(acce_bar(a), C::kEpiWarps * kCta);
    }
    mbar_init(drain_bar, 1);
    mbar_init(report_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmSA)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmSB)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmY)) : "memory");
  }
  if (warp == 1) {
    if (kCta == 1) {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                   "r"(kTmemCols));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    } else {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                   "r"(kTmemCols));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    }
  }
  tc_fence_before();
  __syncthreads();
  if (kCta == 2) cluster_sync();  // both CTAs' barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Launched as a programmatic dependent of the preceding kernel (typically the
  // quantizer that wrote A): the setup above overlapped its tail; nothing below
  // touches global memory before that kernel has completed.
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == 0) {
    // ===================== TMA producer (every CTA) =====================
    {
      Ring st;
      bool ok = true;
      uint32_t issued = 0;  // stages this CTA has issued
      for (int t = pair; t < p.num_tiles && ok; t += npairs) {
        const int m_tile = t / p.n_tiles, n_tile = t % p.n_tiles;
        const int arow = m_tile * C::BM + (int)rank * 128;   // this CTA's A rows
        const int n0 = n_tile * BN;
        const int brow = n0 + (int)rank * C::kBRows;          // this CTA's W rows
        const int ablk = arow / 128;  // this CTA's scale block of A
        const int jb0 = n0 / 128;      // first of the tile's two scale blocks of W
        if constexpr (kPro == 1) {
          // The row block's codes and scales are written by the grid's quantizer warps.
          if (ablk < pq.n_rb && !wait_counter(pq.sync + ablk, 4u * (uint32_t)pq.katoms, abort_flag)) {
            ok = false;
            break;
          }
        }
        for (int kt = 0; kt < p.k_stages; ++kt) {
          if (kCta == 2 && rank == 1 && pair == p.stall_group && p.stall_mode == 2 && issued == 2) {
            // Test hook: this CTA stops loading, as if a wait had timed out, so
            // the pair's loads of the same stage are left half issued.
            atomicOr(&g_device_error, (unsigned)kDevErrTimeout);
            ok = false;
            break;
          }
          if (!__all_sync(0xFFFFFFFFu, wait_bounded(empty_bar(st.slot), st.phase ^ 1u, abort_flag))) {
            ok = false;
            break;
          }
          const uint32_t fb = leader_bar<kCta>(full_bar(st.slot));
          // Scale atoms: one 2048-byte box (the stage's four K=64 atoms, 8-byte
          // elements) of this CTA's A scale block and of the tile's two W scale
          // blocks; blocks and atoms past the arrays read as zero.
          const int sx = kt * kKSteps * (kAtomBytes / 8);
          if (elect_one()) {
            arrive_expect_tx_leader<kCta>(fb, kABytes + C::kBBytes + kSFABytes + kSFBBytes);
            tma_load_2d<kCta>(sbase + C::kOffA + st.slot * kABytes, &tmA, fb, kt * (BK / 2), arow);
            tma_load_2d<kCta>(sbase + C::kOffB + st.slot * C::kBBytes, &tmB, fb, kt * (BK / 2), brow);
            tma_load_2d<kCta>(sbase + C::kOffSFA + st.slot * kSFABytes, &tmSA, fb, sx, ablk);
            tma_load_2d<kCta>(sbase + C::kOffSFB + st.slot * kSFBBytes, &tmSB, fb, sx, jb0);
          }
          __syncwarp();
          st.next(S);
          ++issued;
        }
      }
      // End of loading.  A pair's copies of a stage all complete on the leader's
      // barrier of that stage, which counts one arrival per CTA, so the leader
      // can see every copy of both CTAs land -- once it knows how many stages
      // each CTA issued.  After a timeout the two may have stopped at
      // different stages; the other CTA is told to stop too, the peer reports
      // its count, and the leader arrives in the place of whichever CTA did
      // not issue a stage, so that every issued stage's phase completes when
      // its bytes have landed.  The peer stays resident until the closing
      // cluster barrier, which the leader reaches only after this drain.
      if (kCta == 2 && !ok && lane == 0)
        asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(map_to_rank(smem_u32((const void*)abort_flag), rank ^ 1u)),
                     "r"(1u)
                     : "memory");
      uint32_t last = issued;
      if (kCta == 2 && !leader) {
        if (lane == 0) {
          asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(map_to_rank(smem_u32((const void*)peer_issued), 0)),
                       "r"(issued)
                       : "memory");
          asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(map_to_rank(report_bar, 0))
                       : "memory");
        }
        __syncwarp();
      } else if (kCta == 2) {
        uint32_t reported = issued;
        if (wait_report(report_bar)) reported = *peer_issued;
        const uint32_t lo = min(issued, reported), hi = max(issued, reported);
        if (lane == 0)
          for (uint32_t i = lo; i < hi; ++i)
            asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(full_bar((int)(i % S))) : "memory");
        __syncwarp();
        last = hi;
      }
      if (leader) {
        // The last use of every slot: stage i of slot i % S, phase (i / S) & 1.
        const int slot = (int)(last % S);
        const uint32_t phase = (last / S) & 1u;
        for (int s = 0; s < S; ++s) wait_drain(full_bar(s), (s < slot) ? phase : (phase ^ 1u));
      }
    }
  } else if (warp == 1) {
    // ===================== MMA issuer (leader CTA) =====================
    if (leader) {
      Ring st, sf;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      // Descriptors of stage 0, K step 0; a stage or K step moves the start
      // address field (16-byte units) by a constant.
      const uint64_t adesc0 = smem_desc(sbase + C::kOffA, true);
      const uint64_t bdesc0 = smem_desc(sbase + C::kOffB, true);
      for (int t = pair; t < p.num_tiles && ok; t += npairs) {
        if (!__all_sync(0xFFFFFFFFu, wait_bounded(acce_bar(acc), acc_phase ^ 1u, abort_flag))) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        // A 192-row W tile starts at row 0 or 64 of its first scale block: its
        // W scales start at column 0 or 2 of the 8 copied per K step (a
        // 256-row tile always at 0).
        const uint32_t sfb_shift = (uint32_t)(((t % p.n_tiles) * BN) % 128) / 32u;
        constexpr uint32_t idesc = C::kIdesc;
        for (int kt = 0; kt < p.k_stages; ++kt) {
          const bool landed = wait_bounded(full_bar(st.slot), st.phase, abort_flag);
          if (!__all_sync(0xFFFFFFFFu, landed)) {
            ok = false;
            break;
          }
          if (pair == p.stall_group && p.stall_mode == 1 && t == pair && kt == 3) {
            // Test hook: stop issuing without committing, so every other role
            // of this group runs into its bounded wait and takes the drain path.
            ok = false;
            break;
          }
          tc_fence_after();
          const int ks = min(kKSteps, p.ksteps_total - kt * kKSteps);
          const uint64_t adesc = adesc0 + (uint64_t)((st.slot * kABytes) >> 4);
          const uint64_t bdesc = bdesc0 + (uint64_t)((st.slot * C::kBBytes) >> 4);
          const uint32_t sf_tmem = tmem_base + (uint32_t)(C::kSfCol0 + sf.slot * kSfCols);
          const uint32_t sfa_s = sbase + C::kOffSFA + st.slot * kSFABytes;
          const uint32_t sfb_s = sbase + C::kOffSFB + st.slot * kSFBBytes;
          if (elect_one()) {
            // Scales into this stage's TMEM scale buffer (in every CTA of the
            // group, from its own shared memory), in issue order ahead of the
            // MMAs that read them.
#pragma unroll
            for (int k = 0; k < kKSteps; ++k) {
              tc_cp_atom<kCta>(sf_tmem + 4 * k, smem_desc(sfa_s + k * kAtomBytes, false));
              tc_cp_atom<kCta>(sf_tmem + 4 * kKSteps + 8 * k, smem_desc(sfb_s + k * kAtomBytes, false));
              tc_cp_atom<kCta>(sf_tmem + 4 * kKSteps + 8 * k + 4,
                               smem_desc(sfb_s + (kKSteps + k) * kAtomBytes, false));
            }
            if (ks == kKSteps) {
#pragma unroll
              for (int k = 0; k < kKSteps; ++k)
                tc_mma<kCta>(d_tmem, adesc + (uint64_t)(k * (kMmaK / 2) / 16), bdesc + (uint64_t)(k * (kMmaK / 2) / 16),
                             idesc, (kt | k) != 0 ? 1u : 0u, sf_tmem + 4 * k, sf_tmem + 4 * kKSteps + 8 * k + sfb_shift);
            } else {
              for (int k = 0; k < ks; ++k)
                tc_mma<kCta>(d_tmem, adesc + (uint64_t)(k * (kMmaK / 2) / 16), bdesc + (uint64_t)(k * (kMmaK / 2) / 16),
                             idesc, (kt | k) != 0 ? 1u : 0u, sf_tmem + 4 * k, sf_tmem + 4 * kKSteps + 8 * k + sfb_shift);
            }
            tc_commit<kCta>(empty_bar(st.slot));  // the stage's shared memory (both CTAs), once read
          }
          __syncwarp();
          st.next(S);
          sf.next(kSfBufs);
        }
        if (!ok) break;
        if (elect_one()) tc_commit<kCta>(accf_bar(acc));  // accumulator ready for both CTAs' epilogues
        __syncwarp();
        if (++acc == C::kAccBufs) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      // Drain: every MMA issued above has completed before TMEM is released.
      if (elect_one()) {
        if (kCta == 1)
          tc_commit<1>(drain_bar);
        else
          tc_commit_local2(drain_bar);
      }
      __syncwarp();
      wait_drain(drain_bar, 0);
    }
  } else if (kPro == 1 && warp < C::kEpiWarp0) {
    // ===================== prologue quantizer (every CTA) =====================
    if constexpr (kPro == 1) {
      const QuantTable& tab = *reinterpret_cast<const QuantTable*>(smem + C::kOffQTab);
      const int qw = (int)blockIdx.x * C::kQuantWarps + (warp - 2);
      const int nqw = (int)gridDim.x * C::kQuantWarps;
      const int n_chunks = pq.n_rb * 4 * pq.katoms / kProChunk;
      unsigned long long clips = 0;
      for (int ch = qw; ch < n_chunks; ch += nqw) {
        if (*abort_flag) break;
        const int item0 = ch * kProChunk;
        ProItem cur, nxt;
        pro_load(pq, p.M, item0, lane, cur);
#pragma unroll 1
        for (int k = 0; k < kProChunk; ++k) {
          if (k + 1 < kProChunk) pro_load(pq, p.M, item0 + k + 1, lane, nxt);  // the next item's loads in flight
          pro_quantize_store(pq, tab, p.M, p.K, item0 + k, lane, cur, clips);
          cur = nxt;
        }
        pro_publish(pq, item0 / (4 * pq.katoms), lane);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) clips += __shfl_xor_sync(0xFFFFFFFFu, clips, o);
      if (lane == 0 && clips != 0 && pq.clip != nullptr) atomicAdd(pq.clip, clips);
    }
  } else {
    // ===================== epilogue (every CTA) =====================
    // Warp ew = warp - kEpiWarp0 reads TMEM lane quadrant warp % 4 (32 output
    // rows) and accumulator columns [hcol, hcol + kWarpCols).
    constexpr int kWarpCols = C::kWarpCols;
    constexpr int kChunks = kWarpCols / kEpiCols;
    const int ew = warp - C::kEpiWarp0;
    const int q = warp & 3;
    const int hcol = (ew >> 2) * kWarpCols;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    uint8_t* stage_buf = smem + C::kOffEpi + ew * C::kEpiBufs * kEpiBufBytes;
    uint32_t* bias_s = reinterpret_cast<uint32_t*>(smem + C::kOffBias) + ew * (kWarpCols / 2);  // BF16 pairs
    int acc = 0;
    uint32_t acc_phase = 0;
    int buf = 0;
    unsigned long long clips = 0;  // kEpi == 1: clipped elements of g in this thread's rows
    for (int t = pair; t < p.num_tiles; t += npairs) {
      const int m_tile = t / p.n_tiles, n_tile = t % p.n_tiles;
      const int row0 = m_tile * C::BM + (int)rank * 128 + 32 * q;  // this warp's 32 output rows
      const int n0 = n_tile * BN + hcol;                           // this warp's first column
      // The warp's bias columns (BF16 pairs), staged in its shared memory
      // before the accumulator is ready (8 values per lane).
      if (lane < kWarpCols / 8) {
        uint4 u = make_uint4(0, 0, 0, 0);
        if (p.bias != nullptr && n0 + 8 * lane < p.N)
          u = __ldg(reinterpret_cast<const uint4*>(p.bias + n0 + 8 * lane));
        reinterpret_cast<uint4*>(bias_s)[lane] = u;
      }
      __syncwarp();
      if (!wait_bounded(accf_bar(acc), acc_phase, abort_flag)) break;
      tc_fence_after();
      const uint32_t tcol = tmem_base + lane_base + (uint32_t)(acc * BN + hcol);
      // One 64-column chunk from raw accumulator bits: y = alpha * acc + bias,
      // BF16, then either the quantizing epilogue or a TMA store of y.
      auto emit = [&](const uint32_t(&v)[64], int c) {
        const int col0 = n0 + c * kEpiCols;
        uint32_t packed[32];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const uint2 bw = reinterpret_cast<const uint2*>(bias_s + c * (kEpiCols / 2))[j];
          const float y0 = fmaf(p.alpha, __uint_as_float(v[4 * j]), __uint_as_float(bw.x << 16));
          const float y1 = fmaf(p.alpha, __uint_as_float(v[4 * j + 1]), __uint_as_float(bw.x & 0xFFFF0000u));
          const float y2 = fmaf(p.alpha, __uint_as_float(v[4 * j + 2]), __uint_as_float(bw.y << 16));
          const float y3 = fmaf(p.alpha, __uint_as_float(v[4 * j + 3]), __uint_as_float(bw.y & 0xFFFF0000u));
          packed[2 * j] = pack_bf16x2(y0, y1);
          packed[2 * j + 1] = pack_bf16x2(y2, y3);
        }
        if constexpr (kEpi == 1) {
          // g = GELU(y) per element, then four 16-column blocks of row `row`.
          const QuantTable& qt = *reinterpret_cast<const QuantTable*>(smem + C::kOffEpi);
          const int row = row0 + lane;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            packed[i] = nvfp4::gelu2_bits(packed[i]);
          uint32_t word = 0;
          uint2 cd[4];
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            uint32_t amax;
            const uint32_t sc = nvfp4::quantize_block_codes(qt, eq.inv6sg, packed + 8 * b, amax, cd[b]);
            word |= sc << (8 * b);
            if (row < p.M) clips += nvfp4::block_clips(packed + 8 * b, amax, eq.clip_thr);
          }
          if (row < p.M) {
            uint4* dst = reinterpret_cast<uint4*>(eq.codes + (size_t)row * (size_t)(p.N >> 1) + (col0 >> 1));
            dst[0] = make_uint4(cd[0].x, cd[0].y, cd[1].x, cd[1].y);
            dst[1] = make_uint4(cd[2].x, cd[2].y, cd[3].x, cd[3].y);
          }
          // Scale atom (row / 128, col0 / 64); rows M .. m_pad - 1 get zero scales.
          if (row < eq.m_pad)
            *reinterpret_cast<uint32_t*>(eq.scales + ((size_t)(row >> 7) * eq.katoms + (col0 >> 6)) * 512 +
                                         (row & 31) * 16 + ((row >> 5) & 3) * 4) = row < p.M ? word : 0u;
        } else {
          // Reuse a staging buffer only after its previous TMA store has read it.
          if (lane == 0) {
            if (C::kEpiBufs == 1)
              bulk_wait_read_0();
            else
              bulk_wait_read_1();
          }
          __syncwarp();
          uint8_t* sb = stage_buf + buf * kEpiBufBytes;
          const uint32_t row = (uint32_t)lane;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint32_t chunk = (uint32_t)i ^ (row & 7u);  // 128-byte swizzle
            *reinterpret_cast<uint4*>(sb + row * 128 + chunk * 16) =
                make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && row0 < p.M) tma_store_2d(&tmY, smem_u32(sb), col0, row0);  // rows past M: nothing to store
          if (lane == 0) bulk_commit();
          if (C::kEpiBufs == 2) buf ^= 1;
        }
      };
      auto release = [&]() {  // all TMEM reads of this accumulator are done: hand it back
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_leader<kCta>(leader_bar<kCta>(acce_bar(acc)));
      };
      if constexpr (C::kAccBufs == 1) {
        // One accumulator: copy this warp's columns out, release, then emit.
        uint32_t v[kChunks][64];
#pragma unroll
        for (int c = 0; c < kChunks; ++c) {
          tmem_ld_32(tcol + c * kEpiCols, *reinterpret_cast<uint32_t(*)[32]>(&v[c][0]));
          tmem_ld_32(tcol + c * kEpiCols + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[c][32]));
        }
        tmem_ld_wait_tied(v);
        release();
#pragma unroll
        for (int c = 0; c < kChunks; ++c)
          if (n0 + c * kEpiCols < p.N) emit(v[c], c);  // warp-uniform
      } else {
        for (int c = 0; c < kChunks; ++c) {
          if (n0 + c * kEpiCols >= p.N) break;  // warp-uniform
          uint32_t v[64];
          tmem_ld_32(tcol + c * kEpiCols, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
          tmem_ld_32(tcol + c * kEpiCols + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
          tmem_ld_wait();
          emit(v, c);
        }
        release();
      }
      if (++acc == C::kAccBufs) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (lane == 0) bulk_wait_all();
    if constexpr (kEpi == 1) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) clips += __shfl_xor_sync(0xFFFFFFFFu, clips, o);
      if (lane == 0 && clips != 0 && eq.clip != nullptr) atomicAdd(eq.clip, clips);
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (kCta == 2) cluster_sync();  // the peer no longer needs this CTA's shared memory or TMEM
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    if (kCta == 1)
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols));
    else
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols));
  }
  if constexpr (kPro == 1) {
    // Every producer of this CTA is done with the counters.  The last CTA to
    // get here sets them back to zero for the next launch.
    __shared__ int last_cta;
    if (threadIdx.x == 0) {
      __threadfence();
      last_cta = atomicAdd(pq.sync + pq.n_rb, 1u) == gridDim.x - 1;
    }
    __syncthreads();
    if (last_cta) {
      __threadfence();
      for (int i = threadIdx.x; i <= pq.n_rb; i += blockDim.x) pq.sync[i] = 0u;
    }
  }
}

// Self-test of the bounded wait: one thread waits on an mbarrier that nothing
// arrives on, gives up after limit_ns, and sets the device error word.
__global__ void bounded_wait_selftest_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  abort_flag = 0;
  mbar_init(smem_u32(&bar), 1);
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  wait_bounded(smem_u32(&bar), 0, &abort_flag, limit_ns);
}

// Tensor-pipe rate probe (a measurement, not part of the layer): every CTA pair
// of the grid issues `iters` rounds of four tcgen05.mma cta_group::2
// kind::mxf4nvf4 block_scale (256 x 256 x 64 each, the GEMM's instruction and
// tile) on operands resident in shared memory -- no global memory traffic --
// optionally preceded, as in the GEMM's mainloop, by the twelve tcgen05.cp
// scale copies of a stage into alternating TMEM scale buffers.  Timed by the
// host around the launch, it gives the FP4 tensor rate the GEMM can reach.
constexpr int kProbeThreads = 128;
constexpr int kProbeSmem = 160 * 1024;  // one CTA per SM, so the pairs never wait on each other for TMEM
__global__ void __launch_bounds__(kProbeThreads, 1) mma_rate_probe_kernel(int iters, int with_copies) {
  using C = Cfg<2, 256>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  __shared__ uint64_t done_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t rank = cluster_rank();
  // Operands: A 16 KB, W 16 KB (128-byte swizzled tiles), scale atoms 2 + 4 KB.
  // Pseudo-random codes; scales drawn from E4M3 codes 0x28 .. 0x47 (about 0.25 .. 4).
  for (int i = threadIdx.x; i < (38 * 1024) / 4; i += blockDim.x) {
    uint32_t h = (uint32_t)i * 0x9E3779B1u + (blockIdx.x + 1) * 0x85EBCA6Bu;
    h ^= h >> 15;
    h *= 0x2C1B3C6Du;
    h ^= h >> 12;
    if (i >= 8192) h = 0x28282828u + (h & 0x1F1F1F1Fu);
    reinterpret_cast<uint32_t*>(smem)[i] = h;
  }
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&done_bar), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  fence_proxy_async_smem();
  if ((threadIdx.x >> 5) == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_slot)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;
  if ((threadIdx.x >> 5) == 0 && rank == 0) {
    const uint64_t adesc = smem_desc(sbase, true), bdesc = smem_desc(sbase + kABytes, true);
    const uint32_t sfa_s = sbase + 2 * kABytes, sfb_s = sfa_s + kSFABytes;
    for (int it = 0; it < iters; ++it) {
      const uint32_t sf_tmem = tmem_base + (uint32_t)(C::kSfCol0 + (it & 1) * kSfCols);
      if (elect_one()) {
        if (with_copies || it == 0) {  // without copies, the scales are copied once, before the first round
#pragma unroll
          for (int k = 0; k < kKSteps; ++k) {
            tc_cp_atom<2>(sf_tmem + 4 * k, smem_desc(sfa_s + k * kAtomBytes, false));
            tc_cp_atom<2>(sf_tmem + 4 * kKSteps + 8 * k, smem_desc(sfb_s + k * kAtomBytes, false));
            tc_cp_atom<2>(sf_tmem + 4 * kKSteps + 8 * k + 4, smem_desc(sfb_s + (kKSteps + k) * kAtomBytes, false));
          }
        }
        const uint32_t sf = (with_copies || it == 0) ? sf_tmem : tmem_base + (uint32_t)C::kSfCol0;
#pragma unroll
        for (int k = 0; k < kKSteps; ++k)
          tc_mma<2>(tmem_base, adesc + (uint64_t)(k * (kMmaK / 2) / 16), bdesc + (uint64_t)(k * (kMmaK / 2) / 16),
                    C::kIdesc, (it | k) != 0 ? 1u : 0u, sf + 4 * k, sf + 4 * kKSteps + 8 * k);
      }
      __syncwarp();
    }
    if (elect_one()) tc_commit<2>(smem_u32(&done_bar));  // arrives in both CTAs
    __syncwarp();
  }
  if (threadIdx.x == 0) {
    // Every MMA this pair issued has completed before TMEM is released.
    if (!wait_bounded(smem_u32(&done_bar), 0, &abort_flag)) wait_drain(smem_u32(&done_bar), 0);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  if ((threadIdx.x >> 5) == 1) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols));
  }
}

// ---- host side ----------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  // Looked up once per process (thread-safe static initialization).
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(ptr);
    return nullptr;
  }();
  return fn;
}

// Test hooks (CTA group 0 only): FH_GEMM_TEST_STALL=1 makes the MMA warp stop
// after three stages of its first tile (when K spans at least four stages), so
// that the kernel's bounded waits expire; FH_GEMM_TEST_STALL=2 makes the second
// CTA of the pair stop loading after two stages, so that the two producers end
// at different stages.  Either way the call ends with FH_ERR_TIMEOUT.
int stall_mode() {
  const char* e = getenv("FH_GEMM_TEST_STALL");  // read per launch, so a test can switch it off again
  return (e != nullptr && (e[0] == '1' || e[0] == '2') && e[1] == 0) ? e[0] - '0' : 0;
}

// Which kernel form to run: the CTA pair (default) or single CTAs.  The
// environment variable FH_GEMM_CTAS=1 selects the single-CTA form (both run the
// same arithmetic; the switch exists to compare them).
int cta_mode() {
  static const int mode = []() {
    const char* e = getenv("FH_GEMM_CTAS");
    return (e != nullptr && e[0] == '1') ? 1 : 2;
  }();
  return mode;
}

// Tile width of the CTA-pair form for an N-column output: 256 unless the
// environment variable FH_GEMM_BN (read at first launch) is 192.
int tile_width(int64_t N) {
  static const int forced = []() {
    const char* e = getenv("FH_GEMM_BN");
    return (e != nullptr && strcmp(e, "192") == 0) ? 192 : (e != nullptr && strcmp(e, "256") == 0) ? 256 : 0;
  }();
  if (forced != 0) return forced;
  (void)N;
  return 256;
}

template <int kCta, int kEpi, int kBN, int kPro = 0>
cudaError_t launch_form(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmSA,
                        const CUtensorMap& tmSB, const CUtensorMap& tmY, const Params& p,
                        const typename EpiSel<kEpi>::type& eq, cudaStream_t s,
                        const typename ProSel<kPro>::type& pq = typename ProSel<kPro>::type()) {
  using C = Cfg<kCta, kBN, kPro>;
  static DeviceTable groups_of;  // resident CTA groups of this form, per device
  int dev = 0;
  cudaGetDevice(&dev);
  const int max_groups = per_device(groups_of, dev, [](int) {
    cudaError_t e = cudaFuncSetAttribute(nvfp4_linear_kernel<kCta, kEpi, kBN, kPro>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemAlloc);
    if (e != cudaSuccess) return -(int)e;
    int max_groups = sm_count() / kCta;
    if (kCta == 2) {
      // Clusters that fit at once (an SM left without a partner cannot host one).
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(2 * max_groups);
      cfg.blockDim = dim3(C::kThreads);
      cfg.dynamicSmemBytes = C::kSmemAlloc;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, nvfp4_linear_kernel<2, kEpi, kBN, kPro>, &cfg) == cudaSuccess &&
          clusters > 0)
        max_groups = clusters < max_groups ? clusters : max_groups;
      cudaGetLastError();
    }
    return max_groups > 0 ? max_groups : 1;
  });
  if (max_groups <= 0) return (cudaError_t)(-max_groups);
  // The quantizing prologue spreads its items over every resident pair, so it
  // launches them all even when there are fewer tiles.
  const int groups = (kPro == 1 || p.num_tiles >= max_groups) ? max_groups : p.num_tiles;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  int nattr = 0;
  attr[nattr].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[nattr++].val.programmaticStreamSerializationAllowed = 1;
  if (kCta == 2) {
    attr[nattr].id = cudaLaunchAttributeClusterDimension;
    attr[nattr].val.clusterDim.x = kCta;
    attr[nattr].val.clusterDim.y = 1;
    attr[nattr++].val.clusterDim.z = 1;
  }
  cfg.gridDim = dim3(groups * kCta);
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmemAlloc;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = nattr;
  return cudaLaunchKernelEx(&cfg, nvfp4_linear_kernel<kCta, kEpi, kBN, kPro>, tmA, tmB, tmSA, tmSB, tmY, p, eq, pq);
}

}  // namespace

bool make_tensor_map_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner,
                        uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                        CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_mma_rate_probe(int iters, int with_copies, int* pairs_out, cudaStream_t s) {
  static DeviceTable pairs_of;
  int dev = 0;
  cudaGetDevice(&dev);
  const int pairs = per_device(pairs_of, dev, [](int) {
    cudaError_t e = cudaFuncSetAttribute(mma_rate_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kProbeSmem);
    if (e != cudaSuccess) return -(int)e;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * (sm_count() / 2));
    cfg.blockDim = dim3(kProbeThreads);
    cfg.dynamicSmemBytes = kProbeSmem;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, mma_rate_probe_kernel, &cfg) != cudaSuccess || clusters < 1)
      clusters = sm_count() / 2;
    cudaGetLastError();
    return clusters < sm_count() / 2 ? clusters : sm_count() / 2;
  });
  if (pairs <= 0) return (cudaError_t)(-pairs);
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(kProbeThreads);
  cfg.dynamicSmemBytes = kProbeSmem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  *pairs_out = pairs;
  return cudaLaunchKernelEx(&cfg, mma_rate_probe_kernel, iters, with_copies);
}

cudaError_t launch_bounded_wait_selftest(uint64_t limit_ns, cudaStream_t s) {
  bounded_wait_selftest_kernel<<<1, 32, 0, s>>>(limit_ns);
  return cudaGetLastError();
}

cudaError_t read_and_clear_device_error(unsigned int* bits, cudaStream_t s) {
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return e;
  unsigned int v = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof v);
  if (e != cudaSuccess) return e;
  e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof zero);
  *bits = v;
  return e;
}

namespace {

// Shared by both epilogue modes: tensor maps, tile counts and the launch.
// y is the BF16 output (mode 0) or null (mode 1, outputs in *eq).
cudaError_t launch_linear(const uint8_t* a_codes, const uint8_t* a_scales, float a_g, const uint8_t* w_codes,
                          const uint8_t* w_scales, float w_g, const uint16_t* bias, uint16_t* y, int64_t M,
                          int64_t N, int64_t K, const EpiQuant* eq, cudaStream_t s, const char** why,
                          const ProQuant* pq = nullptr) {
  const int ctas = pq != nullptr ? 2 : cta_mode();
  const int BN = pq != nullptr ? 256 : (ctas == 2 ? tile_width(N) : 192);
  CUtensorMap tmA, tmB, tmY;
  const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
  if (!make_tensor_map_2d(&tmA, CU_TENSOR_MAP_DATA_TYPE_UINT8, a_codes, (uint64_t)K / 2, (uint64_t)M,
                          (uint64_t)K / 2, BK / 2, 128, sw) ||
      !make_tensor_map_2d(&tmB, CU_TENSOR_MAP_DATA_TYPE_UINT8, w_codes, (uint64_t)K / 2, (uint64_t)N,
                          (uint64_t)K / 2, BK / 2, BN / ctas, sw) ||
      (y != nullptr && !make_tensor_map_2d(&tmY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, (uint64_t)N, (uint64_t)M,
                                           (uint64_t)N * 2, kEpiCols, 32, sw))) {
    *why = "cuTensorMapEncodeTiled failed (driver entry point missing or a layout rule violated)";
    return cudaErrorNotSupported;
  }
  // The scale arrays (tensor-core layout) as 2-D tensors of 8-byte elements:
  // one row per 128-row scale block (K / 64 atoms of 512 bytes), boxes of one
  // stage's four atoms -- one block for A, the tile's two for W.
  CUtensorMap tmSA, tmSB;
  const uint64_t sf_row = (uint64_t)(K / kMmaK) * kAtomBytes;
  if (!make_tensor_map_2d(&tmSA, CU_TENSOR_MAP_DATA_TYPE_UINT64, a_scales, sf_row / 8, (uint64_t)((M + 127) / 128),
                          sf_row, kKSteps * kAtomBytes / 8, 1, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tensor_map_2d(&tmSB, CU_TENSOR_MAP_DATA_TYPE_UINT64, w_scales, sf_row / 8, (uint64_t)((N + 127) / 128),
                          sf_row, kKSteps * kAtomBytes / 8, 2, CU_TENSOR_MAP_SWIZZLE_NONE)) {
    *why = "cuTensorMapEncodeTiled failed for the scale arrays";
    return cudaErrorNotSupported;
  }
  if (y == nullptr) tmY = tmA;  // unused by the quantizing epilogue
  Params p;
  p.bias = bias;
  p.alpha = a_g * w_g;
  p.M = (int)M;
  p.N = (int)N;
  p.K = (int)K;
  const int bm = 128 * ctas;
  const int m_tiles = (int)((M + bm - 1) / bm);
  p.n_tiles = (int)((N + BN - 1) / BN);
  p.num_tiles = m_tiles * p.n_tiles;
  p.k_stages = (int)((K + BK - 1) / BK);
  p.ksteps_total = (int)(K / kMmaK);
  p.stall_mode = stall_mode();
  p.stall_group = p.stall_mode != 0 ? 0 : -1;
  if (pq != nullptr) {
    p.stall_group = -1;
    p.stall_mode = 0;
    return launch_form<2, 0, 256, 1>(tmA, tmB, tmSA, tmSB, tmY, p, EpiNone(), s, *pq);
  }
  if (eq == nullptr) {
    const EpiNone none;
    if (ctas == 1) return launch_form<1, 0, 192>(tmA, tmB, tmSA, tmSB, tmY, p, none, s);
    return BN == 256 ? launch_form<2, 0, 256>(tmA, tmB, tmSA, tmSB, tmY, p, none, s)
                     : launch_form<2, 0, 192>(tmA, tmB, tmSA, tmSB, tmY, p, none, s);
  }
  if (ctas == 1) return launch_form<1, 1, 192>(tmA, tmB, tmSA, tmSB, tmY, p, *eq, s);
  return BN == 256 ? launch_form<2, 1, 256>(tmA, tmB, tmSA, tmSB, tmY, p, *eq, s)
                   : launch_form<2, 1, 192>(tmA, tmB, tmSA, tmSB, tmY, p, *eq, s);
}

}  // namespace

cudaError_t launch_nvfp4_linear(const uint8_t* a_codes, const uint8_t* a_scales, float a_g,
                                const uint8_t* w_codes, const uint8_t* w_scales, float w_g,
                                const uint16_t* bias, uint16_t* y, int64_t M, int64_t N, int64_t K,
                                cudaStream_t s, const char** why) {
  return launch_linear(a_codes, a_scales, a_g, w_codes, w_scales, w_g, bias, y, M, N, K, nullptr, s, why);
}

cudaError_t launch_nvfp4_linear_quant_prologue(const uint16_t* x, int64_t ldx, float a_g, const uint8_t* w_codes,
                                               const uint8_t* w_scales, float w_g, const uint16_t* bias, uint16_t* y,
                                               uint8_t* a_codes, uint8_t* a_scales, unsigned long long* clip,
                                               uint32_t* sync, int64_t M, int64_t N, int64_t K, cudaStream_t s,
                                               const char** why) {
  static thread_local ProQuant pq;  // 3 KB: kept off the stack
  memcpy(&pq.tab, &quant_table_for(a_g), sizeof(QuantTable));
  pq.x = x;
  pq.codes = a_codes;
  pq.scales = a_scales;
  pq.clip = clip;
  pq.sync = sync;
  pq.ldx = ldx;
  pq.inv6sg = (float)(1.0 / (6.0 * (double)a_g));
  pq.clip_thr = clip_threshold_bits(a_g);
  pq.katoms = (int)(K / 64);
  pq.n_rb = (int)((M + 127) / 128);
  return launch_linear(a_codes, a_scales, a_g, w_codes, w_scales, w_g, bias, y, M, N, K, nullptr, s, why, &pq);
}

cudaError_t launch_nvfp4_linear_gelu_quant(const uint8_t* a_codes, const uint8_t* a_scales, float a_g,
                                           const uint8_t* w_codes, const uint8_t* w_scales, float w_g,
                                           const uint16_t* bias, float out_g, uint8_t* out_codes,
                                           uint8_t* out_scales, unsigned long long* out_clip, int64_t M,
                                           int64_t N, int64_t K, cudaStream_t s, const char** why) {
  static thread_local EpiQuant eq;  // 2.9 KB: kept off the stack
  memcpy(&eq.tab, &quant_table_for(out_g), sizeof(QuantTable));
  eq.codes = out_codes;
  eq.scales = out_scales;
  eq.clip = out_clip;
  eq.inv6sg = (float)(1.0 / (6.0 * (double)out_g));
  eq.clip_thr = clip_threshold_bits(out_g);
  eq.katoms = (int)(N / 64);
  eq.m_pad = (int)(((M + 127) / 128) * 128);
  return launch_linear(a_codes, a_scales, a_g, w_codes, w_scales, w_g, bias, nullptr, M, N, K, &eq, s, why);
}

}  // namespace fh
