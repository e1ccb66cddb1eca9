/*
 * fh.h -- C ABI of the NVFP4 quantized linear layer for B200 (sm_100a).
 *
 * The layer is the FP4 linear layer that FastH3 runs inside every block of its
 * diffusion transformer:
 *   - FastH3 thread digest (farwalk.ai), tweet 5/8: on Blackwell the
 *     transformer runs in NVFP4;
 *   - FastH3 thread digest (farwalk.ai), tweet 6/8: every FP4 layer is
 *     calibrated on 1,000 prompts so that large activations are not clipped,
 *     where uncalibrated FP4 scales clip in 40 of 42 blocks (worst 137x);
 *   - FastH3 Trim (comfyui-wiki news), "What the ComfyUI repack contains":
 *     each NVFP4 layer carries an activation scale calibrated on 1,000
 *     prompts, 294 calibrated layers in all;
 *   - FastH3 Trim (comfyui-wiki news), "Trim changes": the transformer's
 *     hidden width is 2,688.
 *
 * NVFP4 (the pages name it without defining it; this is the public format):
 * a tensor x is stored as 4-bit E2M1 codes (magnitudes 0, 0.5, 1, 1.5, 2, 3,
 * 4, 6; bit 3 the sign), one unsigned E4M3 block scale S_b per 16 consecutive
 * elements along K, and one FP32 global scale s_g, with x ~ code * S_b * s_g.
 * Rounding is to nearest, ties to the even code, on the exact quotients
 * (S_b = E4M3(amax_b / (6 s_g)), saturating at 448; code = E2M1(x / (S_b s_g)),
 * saturating at 6; the code's sign bit is always the sign bit of x).
 *
 * Conventions for every entry point:
 *   - Pointers named *_dev or documented as device pointers are device memory
 *     owned by the caller; the library allocates nothing and keeps no state
 *     between calls except a per-device property cache and the device error
 *     words that fh_device_status reads.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL is the legacy default
 *     stream) and the call returns without synchronizing, except where stated.
 *   - The return value is an fh_status.  On failure nothing was enqueued and
 *     fh_last_error() (per host thread) describes the cause.
 *   - Host threads: the property caches are per-device tables of atomics,
 *     filled by the first call of an entry point on each device (with that
 *     device current) and only read afterwards, so calls may come from several
 *     host threads at once and a process may drive several devices (up to 64
 *     device ordinals are cached; higher ones are served uncached).  The
 *     quantizer's decision tables are cached per host thread.
 *     fh_nvfp4_linear_host keeps its copy streams per host thread and device.
 *   - Matrices are row-major.  BF16 values are passed as their uint16 bits.
 *   - Inputs must be finite; results for NaN or Inf inputs are unspecified.
 */
#ifndef FH_H_
#define FH_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* fh_stream_t; /* same type as cudaStream_t */

typedef enum {
  FH_OK = 0,
  FH_ERR_INVALID_ARG = 1,       /* null pointer, bad enum, non-finite or <= 0 scale */
  FH_ERR_UNSUPPORTED_SHAPE = 2, /* a size or alignment rule below is violated */
  FH_ERR_CUDA = 3,              /* a CUDA call failed; fh_last_error() has its text */
  FH_ERR_TIMEOUT = 4,           /* a bounded on-chip wait expired (see fh_device_status) */
  FH_ERR_NO_DEVICE = 5          /* the current device is not an sm_100 GPU */
} fh_status;

/* Scale layouts accepted by fh_quantize_act. */
enum {
  /* scales[r * (K/16) + s]: plain row-major [rows, K/16]. */
  FH_SCALES_ROWMAJOR = 0,
  /* The layout the block-scaled tensor-core MMA reads (fh_nvfp4_linear's
   * operand layout).  Rows are padded to a multiple of 128 and K/16 to a
   * multiple of 4.  The matrix is cut into 512-byte atoms of 128 rows x 4
   * scales; atom (r/128, s/4) sits at ((r/128) * ceil(K/64) + s/4) * 512;
   * inside it, row r%128 = r0 + 32*r1 and scale s%4 = k0 sit at byte
   * r0*16 + r1*4 + k0.  Padding rows hold zero scales. */
  FH_SCALES_MMA_TILED = 1
};

/* Library version, as major*10000 + minor*100 + patch. */
int fh_version(void);

/* Text of the last failure on this host thread ("" if none). */
const char* fh_last_error(void);

/* Global scale from a calibrated amax (host only, no GPU needed).
 * Calibration maps the amax seen over the calibration set onto the largest
 * magnitude of the scaled format, 6 * 448 = 2688, so that no calibrated
 * activation clips (FastH3 thread digest, tweet 6/8).  Returns the SMALLEST
 * FP32 s_g with 2688 * s_g >= amax; amax == 0 gives 1.0; a negative or
 * non-finite amax gives NaN. */
float fh_scale_from_amax(float amax);

/* Bytes of the scale array of a quantized [rows, K] matrix in `layout`
 * (0 for an invalid layout or size). */
size_t fh_scales_bytes(int64_t rows, int64_t K, int layout);

/* Running max |x| over a BF16 matrix x [rows, cols] (leading dimension ldx >=
 * cols, in elements), merged into *amax_dev (device float, caller initialises
 * it, e.g. to 0): *amax_dev = max(*amax_dev, max |x|).  Calling it once per
 * calibration batch gives the calibrated amax (FastH3 thread digest, tweet
 * 6/8).  Exact (a max), deterministic.  rows == 0 or cols == 0 enqueues
 * nothing.  Requires 0 <= rows, cols and ldx >= cols. */
int fh_amax(const uint16_t* x_dev, int64_t rows, int64_t cols, int64_t ldx,
            float* amax_dev, fh_stream_t stream);

/* NVFP4 quantization of BF16 activations (or weights) x [M, K] (leading
 * dimension ldx >= K, elements) with the calibrated global scale s_g
 * (FastH3 Trim, "What the ComfyUI repack contains": per-layer calibrated
 * activation scale).
 * Outputs (device memory, caller-allocated):
 *   codes       [M, K/2] bytes; element 2j of a row in the low nibble of byte j.
 *   scales      E4M3 block scales in `scale_layout`
 *               (fh_scales_bytes(M, K, scale_layout) bytes).
 *   clip_count  device counter, INCREMENTED by the number of elements with
 *               |x| > 2688 * s_g (beyond the largest magnitude the scaled
 *               format holds; FastH3 thread digest, tweet 6/8); may be NULL.
 * Requires: M >= 0, K > 0, K % 16 == 0 (K % 64 == 0 for FH_SCALES_MMA_TILED),
 * ldx >= K and ldx % 8 == 0, x_dev and codes_dev 16-byte aligned, s_g finite
 * and > 0.  Results are bit-exact with the rounding rules in the header
 * comment.  M == 0 only pads nothing and enqueues nothing. */
int fh_quantize_act(const uint16_t* x_dev, int64_t M, int64_t K, int64_t ldx,
                    float global_scale, uint8_t* codes_dev, uint8_t* scales_dev,
                    unsigned long long* clip_count_dev, int scale_layout,
                    fh_stream_t stream);

/* NVFP4 quantization of GELU(x) for BF16 x [M, K] (leading dimension ldx):
 * the FFN's activation applied while quantizing the down projection's input,
 * so GELU(x) is never written.  Bit-identical to fh_gelu_bf16 followed by
 * fh_quantize_act with FH_SCALES_MMA_TILED (same GELU arithmetic, same
 * rounding rules); outputs and clip count as for fh_quantize_act.  Requires
 * K % 64 == 0, ldx >= K, ldx % 8 == 0, 16-byte aligned pointers, s_g finite
 * and > 0. */
int fh_gelu_quantize_act(const uint16_t* x_dev, int64_t M, int64_t K, int64_t ldx, float global_scale,
                         uint8_t* codes_dev, uint8_t* scales_dev, unsigned long long* clip_count_dev,
                         fh_stream_t stream);

/* NVFP4 linear layer on the tcgen05 tensor cores (FastH3 thread digest, tweet
 * 5/8: the transformer's linear layers in NVFP4 on Blackwell):
 *   y[m, n] = bf16( a_gscale * w_gscale * sum_k A[m,k] * W[n,k] + bias[n] )
 * where A[m,k] = E2M1(a_codes) * E4M3(a_scales) and W likewise, both K-major
 * (W is [N, K], the usual nn.Linear weight), the block products are summed in
 * FP32 on the tensor cores, and the epilogue is one FP32 fma then a
 * round-to-nearest-even BF16 store.
 *   a_codes  [M, K/2], a_scales FH_SCALES_MMA_TILED of [M, K]
 *   w_codes  [N, K/2], w_scales FH_SCALES_MMA_TILED of [N, K]
 *   bias     [N] BF16 or NULL; y [M, N] BF16 (row stride N).
 * Requires: M, N >= 0, K > 0, K % 64 == 0, N % 8 == 0, all pointers 16-byte
 * aligned, scales finite and > 0.  M == 0 or N == 0 enqueues nothing.
 * A bounded wait that expires inside the kernel sets the device error word
 * (see fh_device_status) instead of hanging; the kernel then drains the
 * copies and MMAs it issued and frees its TMEM before it exits.
 * Environment: FH_GEMM_CTAS=1 (read at the first launch) selects the
 * single-CTA form (128-row tiles) instead of the CTA pair; FH_GEMM_BN=192
 * (read at the first launch) makes the CTA pair use 256 x 192 tiles instead
 * of the default 256 x 256 (both give identical results);
 * FH_GEMM_TEST_STALL=1 (read at each launch) is a test hook that makes the
 * first CTA group's MMA warp stop after three stages of its first tile
 * (K >= 1024), and FH_GEMM_TEST_STALL=2 one that makes the second CTA of the
 * first pair stop loading after two stages; either call ends with
 * FH_ERR_TIMEOUT after draining what it issued. */
int fh_nvfp4_linear(const uint8_t* a_codes_dev, const uint8_t* a_scales_dev, float a_gscale,
                    const uint8_t* w_codes_dev, const uint8_t* w_scales_dev, float w_gscale,
                    const uint16_t* bias_dev, uint16_t* y_dev, int64_t M, int64_t N,
                    int64_t K, fh_stream_t stream);

/* The NVFP4 linear layer with the quantization of its BF16 input fused into
 * the same kernel (FastH3 Trim, "How fast it runs": the FP8 path's fused
 * per-tensor kernel; FastH3 thread digest, tweet 6/8: every FP4 layer's input
 * quantized with its calibrated scale).  Computes exactly fh_quantize_act
 * (FH_SCALES_MMA_TILED) followed by fh_nvfp4_linear, with byte-identical
 * results, in one launch: two warps of every CTA quantize x while the tensor
 * cores multiply the row blocks already quantized, so the quantization runs
 * under the GEMM instead of before it.
 *   x          BF16 [M, K], rows ldx elements apart (ldx >= K, ldx % 8 == 0)
 *   a_codes, a_scales  outputs: x's codes [M, K/2] and tensor-core-layout
 *              scales (fh_scales_bytes(M, K, FH_SCALES_MMA_TILED) bytes), as
 *              fh_quantize_act writes them; the GEMM reads them back from L2
 *   clip_count device counter, incremented as by fh_quantize_act (may be NULL)
 *   sync       fh_nvfp4_linear_fused_quant_sync_bytes(M) bytes of device
 *              scratch the caller owns: ceil(M/128) row-block ready counters
 *              and an exit counter.  It must be zero before the first call
 *              (e.g. cudaMemsetAsync); every call leaves it zero again,
 *              including a call that ends with FH_ERR_TIMEOUT.  Calls that
 *              overlap on the GPU must use different sync buffers.
 *   w_codes, w_scales, bias, y, N  as for fh_nvfp4_linear.
 * Requires K % 64 == 0, N % 8 == 0, 16-byte aligned pointers (sync 4-byte).
 * The kernel's CTAs wait on one another (a row block is quantized by other
 * CTAs than the ones that multiply it), so the grid is sized to the CTA pairs
 * that fit on the device at once; if other work keeps SMs busy for seconds,
 * the bounded waits expire and the call reports FH_ERR_TIMEOUT through
 * fh_device_status instead of hanging. */
int fh_nvfp4_linear_fused_quant(const uint16_t* x_dev, int64_t M, int64_t K, int64_t ldx, float a_gscale,
                                const uint8_t* w_codes_dev, const uint8_t* w_scales_dev, float w_gscale,
                                const uint16_t* bias_dev, uint16_t* y_dev, int64_t N, uint8_t* a_codes_dev,
                                uint8_t* a_scales_dev, unsigned long long* clip_count_dev, uint32_t* sync_dev,
                                fh_stream_t stream);

/* Bytes of the sync scratch fh_nvfp4_linear_fused_quant needs for M rows
 * (0 for M < 0 or M >= 2^31). */
size_t fh_nvfp4_linear_fused_quant_sync_bytes(int64_t M);

/* The NVFP4 linear layer fused with the activation that follows it and with
 * the quantization of the next layer's input: the FFN's up projection, whose
 * output feeds the down projection (FastH3 thread digest, tweet 5/8: the
 * transformer's linear layers run in NVFP4; tweet 6/8: each FP4 layer's input
 * is quantized with its calibrated scale).  For every output element,
 *   y = bf16( a_gscale * w_gscale * sum_k A[m,k] * W[n,k] + bias[n] )
 *   g = bf16( y/2 * erfc(-y / sqrt 2) )        (exact-erf GELU in FP32)
 * exactly as fh_nvfp4_linear followed by fh_gelu_bf16 would compute them, and
 * g is quantized with the next layer's global scale out_gscale exactly as
 * fh_quantize_act does (FH_SCALES_MMA_TILED layout):
 *   out_codes  [M, N/2], out_scales FH_SCALES_MMA_TILED of [M, N] (padding
 *   rows zero), *out_clip_count_dev += elements with |g| > 2688 * out_gscale
 *   (out_clip_count_dev may be NULL).
 * y and g never reach memory: the BF16 intermediate of M * N * 2 bytes is not
 * written or read.  The outputs are bit-identical to the three separate calls.
 * Requires everything fh_nvfp4_linear requires, N % 64 == 0, out_gscale finite
 * and > 0, out_codes_dev and out_scales_dev 16-byte aligned. */
int fh_nvfp4_linear_gelu_quant(const uint8_t* a_codes_dev, const uint8_t* a_scales_dev, float a_gscale,
                               const uint8_t* w_codes_dev, const uint8_t* w_scales_dev, float w_gscale,
                               const uint16_t* bias_dev, float out_gscale, uint8_t* out_codes_dev,
                               uint8_t* out_scales_dev, unsigned long long* out_clip_count_dev,
                               int64_t M, int64_t N, int64_t K, fh_stream_t stream);

/* The layer on host buffers: y_host = bf16(a_g * w_g * Q(x_host) . W^T + bias),
 * quantizing x with a_gscale exactly as fh_quantize_act and multiplying as
 * fh_nvfp4_linear, so y_host is byte-identical to those two calls on the same
 * rows.  x_host: BF16 [M, K] in host memory; y_host: BF16 [M, N] in host memory,
 * written; both should be page-locked (cudaHostAlloc / cudaHostRegister) --
 * pageable memory works, but then the copies do not overlap.  Weights, bias and
 * the clip counter (may be NULL) are device memory as in fh_nvfp4_linear.
 * The rows are processed in chunks of chunk_rows (a multiple of 128): each
 * chunk's quantization and GEMM run on `stream`, while the next chunk's upload
 * and the previous chunk's download run on two copy streams, so transfers in
 * both directions and the kernels overlap.  The call is ordered on `stream`
 * like any other: the copies start after the work enqueued there before the
 * call, and work enqueued there afterwards sees y_host complete (synchronize
 * before reading it on the host).
 * workspace_dev: device memory owned by the caller, 256-byte aligned, at least
 * fh_nvfp4_linear_host_workspace_bytes(K, N, chunk_rows) bytes (two x chunks,
 * the chunk's codes and scales, two y chunks), not used by other work while
 * the call runs; the library allocates no device memory.  The exception to the
 * "allocates nothing" convention: on the first call from a host thread on a
 * device, the library creates that thread's two copy streams and eleven events
 * for the device, kept until the process exits.
 * Failure: argument errors enqueue nothing.  A CUDA error in the middle of the
 * chunk loop returns FH_ERR_CUDA after part of the work was enqueued; that
 * work stays ordered on `stream` (the copy streams are joined back into it
 * before the call returns), so synchronize `stream` before freeing x_host,
 * y_host or the workspace.
 * Shape rules as fh_nvfp4_linear (K % 64 == 0, N % 8 == 0). */
int fh_nvfp4_linear_host(const uint16_t* x_host, int64_t M, int64_t K, float a_gscale, const uint8_t* w_codes_dev,
                         const uint8_t* w_scales_dev, float w_gscale, const uint16_t* bias_dev, int64_t N,
                         uint16_t* y_host, unsigned long long* clip_count_dev, int64_t chunk_rows,
                         void* workspace_dev, size_t workspace_bytes, fh_stream_t stream);

/* Workspace bytes fh_nvfp4_linear_host needs for K, N and chunk_rows; 0 if the
 * shape is not supported. */
size_t fh_nvfp4_linear_host_workspace_bytes(int64_t K, int64_t N, int64_t chunk_rows);

/* Bytes of the library's static device scratch array (16 MiB). */
#define FH_NOALLOC_SCRATCH_BYTES (16u << 20)

/* The layer on host buffers without any device allocation, for callers that
 * cannot allocate device memory: a serving engine or host application that
 * reserves the device's memory for its own pool up front, a plugin that may
 * only use memory handed to it, or a caller that must not pay for cudaMalloc /
 * cudaFree, which can synchronize the device.  The pages have no counterpart;
 * this is a packaging of fh_nvfp4_linear_host.
 * Computes the same y_host as fh_nvfp4_linear_host, byte for byte, but stages
 * its row chunks in a scratch array that is part of the library's own device
 * memory (FH_NOALLOC_SCRATCH_BYTES per device, held by every device on which
 * the library's module is loaded until the process exits) instead of a
 * caller's workspace.  The library calls no cudaMalloc or cudaFree here.
 * Each chunk (the largest multiple of 128 rows whose x, codes, scales and
 * output fit the array) is uploaded, quantized, multiplied and downloaded in
 * order on `stream`; nothing overlaps inside a call.
 * The first call on a device looks up the array's device address with that
 * device current and keeps it; make that first call before any stream capture.
 * Every call on a device shares the one array, and each call rewrites
 * everything it reads from it, so the contents a previous call left are never
 * used.  Calls whose work overlaps on the GPU (calls on two streams, or from
 * two host threads, of one process) race on the array and corrupt each
 * other's results: serialize them, for example on one stream.
 * x_host, y_host, weights, bias and clip counter as for fh_nvfp4_linear_host.
 * Requires K % 64 == 0, N % 8 == 0, and that one 128-row chunk fits the array:
 * 128 * (2.5625 * K + 2 * N) bytes, plus alignment, at most
 * FH_NOALLOC_SCRATCH_BYTES (FH_ERR_UNSUPPORTED_SHAPE otherwise, e.g.
 * K = N = 2688 gives 1280-row chunks, K = 10752 with N = 2688 384-row ones).
 * A CUDA error in the chunk loop returns FH_ERR_CUDA after part of the work was
 * enqueued on `stream`; synchronize it before freeing the buffers. */
int fh_nvfp4_linear_host_noalloc(const uint16_t* x_host, int64_t M, int64_t K, float a_gscale,
                                 const uint8_t* w_codes_dev, const uint8_t* w_scales_dev, float w_gscale,
                                 const uint16_t* bias_dev, int64_t N, uint16_t* y_host,
                                 unsigned long long* clip_count_dev, fh_stream_t stream);

/* Permute FH_SCALES_MMA_TILED scales of a [rows, K] matrix into row-major
 * [rows, K/16] (drops the padding).  Requires K % 64 == 0. */
int fh_scales_to_rowmajor(const uint8_t* tiled_dev, uint8_t* rowmajor_dev, int64_t rows,
                          int64_t K, fh_stream_t stream);

/* Exact-erf GELU on BF16, y = bf16(x/2 * (1 + erf(x/sqrt 2))), evaluated in
 * FP32 as x/2 * erfc(-x/sqrt 2) (no cancellation for negative x), with erfc
 * from a Chebyshev-fitted approximation of fractional error below 1.2e-7 (far
 * below BF16's 2^-8); the activation between the two linear layers of the
 * FFN.  n >= 0; x_dev and y_dev 16-byte aligned; in-place (x_dev == y_dev)
 * is allowed. */
int fh_gelu_bf16(const uint16_t* x_dev, uint16_t* y_dev, int64_t n, fh_stream_t stream);

/* INT8 query/key quantization for attention scores.  FastH3 Trim
 * (comfyui-wiki news), "How fast it runs": where no FP4 tensor cores exist,
 * the query and the key are quantized to INT8 for the score computation.  The
 * pages fix neither the granularity nor the rounding; this library takes one
 * symmetric scale per row (one token of one head), in IEEE FP32:
 *   s = amax_row / 127,   q = clamp(round_half_even(x / s), -127, 127),
 * with s = 0 and q = 0 for an all-zero row.
 * x_dev: BF16 [rows, d], rows ldx elements apart; q_dev: int8 [rows, d], dense
 * (rows d bytes apart); scales_dev: FP32 [rows].  rows >= 0, d > 0, d % 8 == 0,
 * ldx >= d, ldx % 8 == 0; x_dev and q_dev 16-byte aligned, scales_dev 4-byte
 * aligned.  Bit-exact: every decision is one IEEE single division. */
int fh_quantize_int8_rows(const uint16_t* x_dev, int64_t rows, int64_t d, int64_t ldx, int8_t* q_dev,
                          float* scales_dev, fh_stream_t stream);

/* Attention scores from INT8 queries and keys (same passage as above):
 *   S[h, i, j] = (float(acc) * (s_q[h, i] * sm_scale)) * s_k[h, j],
 *   acc = sum_c q[h, i, c] * k[h, j, c]   (exact INT32 on the tensor cores),
 * every product an FP32 multiply rounded to nearest.
 * q_dev: int8 [heads, tq, d]; k_dev: int8 [heads, tk, d]; q_scales_dev FP32
 * [heads, tq]; k_scales_dev FP32 [heads, tk] (the outputs of
 * fh_quantize_int8_rows over the flattened rows); s_dev: FP32 [heads, tq, tk],
 * every element written.  heads, tq, tk >= 0 (each below 2^31); d > 0,
 * d % 16 == 0, d <= 65536 (any tk; tk % 4 == 0 takes 16-byte stores); q_dev, k_dev and s_dev 16-byte
 * aligned; sm_scale finite.  A bounded wait that expires sets the device error
 * word (fh_device_status) and the kernel drains and returns.
 * Environment: FH_INT8_TEST_STALL=1 (read at each launch) is a test hook that
 * makes the first CTA's MMA warp stop before its first MMA, so the call ends
 * with FH_ERR_TIMEOUT after about 4 s. */
int fh_int8_attention_scores(const int8_t* q_dev, const float* q_scales_dev, const int8_t* k_dev,
                             const float* k_scales_dev, float sm_scale, float* s_dev, int64_t heads, int64_t tq,
                             int64_t tk, int64_t d, fh_stream_t stream);

/* AdaLN timestep conditioning through a shared low-rank basis.  FastH3 Trim
 * (comfyui-wiki news), "What Trim changes": AdaLN maps the 2,688-wide time
 * embedding to six modulation vectors per block; Trim replaces the per-block
 * projections with one shared 2,688 -> 16 basis and a small projection per
 * block, stored in FP16.  This call evaluates both maps, linear, in FP32:
 *   code[b, j]   = sum_k basis[j, k] * temb[b, k]
 *   mod[l, b, i] = sum_j proj[l, i, j] * code[b, j] + bias[l, i]
 * temb_dev: BF16 [bt, d]; basis_dev: FP16 [r, d]; proj_dev: FP16 [blocks, n, r];
 * bias_dev: FP16 [blocks, n] or NULL (no bias); code_dev: FP32 [bt, r], written
 * (the shared code, an output the caller owns); mod_dev: FP32 [blocks, bt, n],
 * written (for the pages' model n = 6 * 2688, the six modulation vectors of a
 * block side by side).  bt, blocks, n >= 0 (blocks * n < 2^31); d > 0,
 * d % 8 == 0; r in {8, 16, 24, 32}; temb, basis and proj 16-byte aligned, bias
 * 2-byte, code and mod 4-byte.  The result is within the FP32 dot-product bound
 * of the exact value; it is exact when every partial sum is representable.
 * Two kernels run on `stream`, the second launched as a programmatic
 * dependent of the first. */
int fh_adaln_modulation(const uint16_t* temb_dev, int64_t bt, int64_t d, const uint16_t* basis_dev, int64_t r,
                        const uint16_t* proj_dev, const uint16_t* bias_dev, int64_t blocks, int64_t n,
                        float* code_dev, float* mod_dev, fh_stream_t stream);

/* Diagnostic of the failure path: enqueues a one-thread kernel whose bounded
 * mbarrier wait (the same wait every pipeline stage of fh_nvfp4_linear uses)
 * can never be satisfied and gives up after limit_us microseconds (1 .. 2e6),
 * setting the device error word.  A following fh_device_status returns
 * FH_ERR_TIMEOUT and the CUDA context stays usable.  The pages describe no
 * failure handling; this exists so the timeout path can be tested without
 * hanging or faulting a GPU. */
int fh_selftest_bounded_wait(uint32_t limit_us, fh_stream_t stream);

/* Measurement of the FP4 tensor rate, not part of the layer (the pages give no
 * kernel-level figures): enqueues one CTA pair per pair of SMs, each issuing
 * `iters` rounds of four tcgen05.mma cta_group::2 kind::mxf4nvf4 block_scale
 * instructions of 256 x 256 x 64 -- the instruction and tile of
 * fh_nvfp4_linear -- on operands resident in shared memory, so no global
 * memory is touched.  with_scale_copies != 0 precedes every round with the
 * twelve tcgen05.cp scale-atom copies the GEMM issues per 256-deep K stage.
 * Each round is 2 * 256 * 256 * 256 FLOP per pair; time the call with events
 * on `stream`.  *pairs_out (host) receives the number of pairs launched.
 * 1 <= iters <= 1e6 (about 0.3 s at most). */
int fh_selftest_mma_rate(int32_t iters, int32_t with_scale_copies, int32_t* pairs_out, fh_stream_t stream);

/* Synchronizes `stream`, then reads and clears the device error word of the
 * current device.  Returns FH_OK, FH_ERR_TIMEOUT if a kernel gave up on a
 * bounded wait since the last call, or FH_ERR_CUDA. */
int fh_device_status(fh_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FH_H_ */
