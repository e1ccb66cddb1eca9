// fh_internal.h -- declarations shared by the CUDA translation units of libfh.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/fh.h"
#include "fh_nvfp4.cuh"

namespace fh {

// Device error word bits (read and cleared by fh_device_status).
enum : unsigned int {
  kDevErrTimeout = 1u,  // a bounded mbarrier wait expired
};

// Host side: synchronize `s`, then read and clear the device error word of the
// current device (fh_gemm.cu owns the word).
cudaError_t read_and_clear_device_error(unsigned int* bits, cudaStream_t s);
// The quantizer's error word (fh_quant.cu); call after the stream is synchronized.
cudaError_t read_and_clear_quant_error(unsigned int* bits);

// The INT8 score kernel's error word (fh_int8.cu); call after the stream is synchronized.
cudaError_t read_and_clear_int8_error(unsigned int* bits);

// Per-device caches of the host side.  Each table holds one int per device
// ordinal, 0 meaning "not filled yet"; the first call on a device fills its
// entry with the device current.  Entries are atomics, so host threads may
// race on the first fill: each computes the same value and the last store
// wins.  Devices beyond the table are served uncached.
constexpr int kMaxDevices = 64;
using DeviceTable = std::atomic<int>[kMaxDevices];

// The value for device `dev` from `table`, computing it with fill(dev) on the
// first use.  fill returns a value > 0, or <= 0 for a failure, which is
// returned without being cached.
template <class F>
int per_device(DeviceTable& table, int dev, F fill) {
  if (dev < 0 || dev >= kMaxDevices) return fill(dev);
  int v = table[dev].load(std::memory_order_acquire);
  if (v == 0) {
    v = fill(dev);
    if (v > 0) table[dev].store(v, std::memory_order_release);
  }
  return v;
}

// Number of SMs of the current device (cached per device).
int sm_count();

// 2-D tiled tensor map of a row-major matrix (inner extent `inner` elements,
// `outer` rows, rows `row_bytes` apart) with a box of box_inner x box_outer
// elements; out-of-range elements of a box read as zero.  False if the driver
// entry point is missing or a layout rule is violated (fh_gemm.cu).
bool make_tensor_map_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner,
                        uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                        CUtensorMapSwizzle swizzle);

// Exact decision table of the NVFP4 quantizer for global scale sg (host, cached
// per thread), and the BF16 bits of the smallest magnitude strictly beyond
// 2688 sg (the clip threshold) (fh_quant.cu).
const QuantTable& quant_table_for(float sg);
uint32_t clip_threshold_bits(float sg);

// Quantizer / calibration / glue launchers (fh_quant.cu).  Arguments are
// validated by the caller.
// gelu: quantize GELU(x) (tensor-core scale layout only).
cudaError_t launch_quantize(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, float sg,
                            uint8_t* codes, uint8_t* scales, unsigned long long* clip,
                            int layout, bool gelu, cudaStream_t s);
cudaError_t launch_amax(const uint16_t* x, int64_t rows, int64_t cols, int64_t ldx, float* amax,
                        cudaStream_t s);
cudaError_t launch_scales_to_rowmajor(const uint8_t* tiled, uint8_t* rowmajor, int64_t rows,
                                      int64_t K, cudaStream_t s);
cudaError_t launch_gelu(const uint16_t* x, uint16_t* y, int64_t n, cudaStream_t s);

// Tensor-pipe rate probe (fh_gemm.cu): every resident CTA pair issues `iters`
// rounds of four 256 x 256 x 64 block-scaled FP4 MMAs from shared memory
// (with_copies: each round preceded by the GEMM's twelve scale copies);
// *pairs_out receives the number of pairs launched.
cudaError_t launch_mma_rate_probe(int iters, int with_copies, int* pairs_out, cudaStream_t s);

// One-thread kernel whose bounded wait runs out after limit_ns (fh_gemm.cu).
cudaError_t launch_bounded_wait_selftest(uint64_t limit_ns, cudaStream_t s);

// GEMM launcher (fh_gemm.cu).  Returns a CUDA error, or cudaErrorNotSupported
// when the tensor maps cannot be built (message in *why).
cudaError_t launch_nvfp4_linear(const uint8_t* a_codes, const uint8_t* a_scales, float a_g,
                                const uint8_t* w_codes, const uint8_t* w_scales, float w_g,
                                const uint16_t* bias, uint16_t* y, int64_t M, int64_t N,
                                int64_t K, cudaStream_t s, const char** why);

// The same GEMM with the epilogue that emits the next layer's NVFP4 input:
// GELU(bf16(alpha * acc + bias)) quantized with global scale out_g into
// out_codes [M, N/2] and tensor-core-layout out_scales of [M, N]; clipped
// elements are added to *out_clip (if not null).  Requires N % 64 == 0.
cudaError_t launch_nvfp4_linear_gelu_quant(const uint8_t* a_codes, const uint8_t* a_scales, float a_g,
                                           const uint8_t* w_codes, const uint8_t* w_scales, float w_g,
                                           const uint16_t* bias, float out_g, uint8_t* out_codes,
                                           uint8_t* out_scales, unsigned long long* out_clip, int64_t M,
                                           int64_t N, int64_t K, cudaStream_t s, const char** why);

// The GEMM with the activations' quantization fused into the kernel: x BF16
// [M, K] (rows ldx elements apart) is quantized with global scale a_g by two
// warps of every CTA into a_codes [M, K/2] and tensor-core-layout a_scales
// (outputs), which the same kernel's tiles read once each row block is done;
// sync: ceil(M / 128) + 1 words, zero at launch and zero again at exit.
// Clipped elements of x are added to *clip (if not null).
cudaError_t launch_nvfp4_linear_quant_prologue(const uint16_t* x, int64_t ldx, float a_g, const uint8_t* w_codes,
                                               const uint8_t* w_scales, float w_g, const uint16_t* bias, uint16_t* y,
                                               uint8_t* a_codes, uint8_t* a_scales, unsigned long long* clip,
                                               uint32_t* sync, int64_t M, int64_t N, int64_t K, cudaStream_t s,
                                               const char** why);

// INT8 query/key path (fh_int8.cu).  Arguments are validated by the caller.
// Per-row symmetric INT8 quantization of BF16 rows (d % 8 == 0).
cudaError_t launch_int8_quantize_rows(const uint16_t* x, int64_t rows, int64_t d, int64_t ldx, int8_t* q,
                                      float* scales, cudaStream_t s);
// S[h, i, j] = (float(q_i . k_j) * (s_q[i] * sm_scale)) * s_k[j] in FP32 for
// q [heads, tq, d], k [heads, tk, d] INT8 and out [heads, tq, tk] FP32 (d % 16 == 0,
// tk % 4 == 0).  cudaErrorNotSupported with a message in *why when the tensor
// maps cannot be built.
cudaError_t launch_int8_scores(const int8_t* q, const float* q_scales, const int8_t* k, const float* k_scales,
                               float sm_scale, float* out, int64_t heads, int64_t tq, int64_t tk, int64_t d,
                               cudaStream_t s, const char** why);

// AdaLN basis projection (fh_adaln.cu): code [bt, r] = e . basis^T, then
// mod [L, bt, n] = proj . code^T + bias, in FP32 from BF16 e and FP16 weights.
// r in {8, 16, 24, 32}; d % 8 == 0.  Arguments are validated by the caller.
cudaError_t launch_adaln_modulation(const uint16_t* e, int64_t bt, int64_t d, const uint16_t* basis, int64_t r,
                                    const uint16_t* proj, const uint16_t* bias, int64_t L, int64_t n, float* code,
                                    float* mod, cudaStream_t s);

// The layer on host buffers, pipelined over row chunks (fh_host.cu).  Arguments
// are validated by the caller; the workspace holds host_linear_workspace_bytes.
size_t host_linear_workspace_bytes(int64_t K, int64_t N, int64_t chunk_rows);
cudaError_t launch_nvfp4_linear_host(const uint16_t* x_host, int64_t M, int64_t K, float a_g, const uint8_t* w_codes,
                                     const uint8_t* w_scales, float w_g, const uint16_t* bias, int64_t N,
                                     uint16_t* y_host, unsigned long long* clip, int64_t chunk_rows, void* workspace,
                                     cudaStream_t s, const char** why);

// The host-buffer layer staged in the library's static scratch array
// (fh_noalloc.cu).  noalloc_chunk_rows: rows per chunk for K and N (a multiple
// of 128), 0 if not even 128 rows fit; noalloc_chunk_bytes: scratch bytes one
// chunk of that many rows uses.  Arguments are validated by the caller.
int64_t noalloc_chunk_rows(int64_t K, int64_t N);
size_t noalloc_chunk_bytes(int64_t K, int64_t N, int64_t rows);
cudaError_t launch_nvfp4_linear_host_noalloc(const uint16_t* x_host, int64_t M, int64_t K, float a_g,
                                             const uint8_t* w_codes, const uint8_t* w_scales, float w_g,
                                             const uint16_t* bias, int64_t N, uint16_t* y_host,
                                             unsigned long long* clip, cudaStream_t s, const char** why);

}  // namespace fh
