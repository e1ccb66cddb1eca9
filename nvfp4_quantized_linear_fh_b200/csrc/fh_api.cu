// fh_api.cu -- the extern "C" entry points declared in include/fh.h: argument
// validation, error reporting and dispatch to the kernels.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "fh_internal.h"

namespace {

thread_local char g_last_error[512] = "";

int fail(int status, const char* fmt, const char* detail = nullptr) {
  snprintf(g_last_error, sizeof g_last_error, fmt, detail ? detail : "");
  return status;
}

int cuda_fail(cudaError_t e, const char* where) {
  snprintf(g_last_error, sizeof g_last_error, "%s: %s", where, cudaGetErrorString(e));
  return FH_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device checks shared by every entry point: a current device of compute
// capability 10.0 (B200 class).  Cached per device.
int check_device() {
  static fh::DeviceTable checked;
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  const int ok = fh::per_device(checked, dev, [](int d) {
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, d);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, d);
    return (major == 10 && minor == 0) ? 1 : -1;
  });
  if (ok <= 0) return fail(FH_ERR_NO_DEVICE, "current device is not an sm_100 GPU%s");
  return FH_OK;
}

}  // namespace

namespace fh {

int sm_count() {
  static DeviceTable counts;
  int dev = 0;
  cudaGetDevice(&dev);
  const int count = per_device(counts, dev, [](int d) {
    int c = 0;
    cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, d);
    return c;
  });
  return count > 0 ? count : 1;
}

}  // namespace fh

extern "C" {

int fh_version(void) { return 10000; }

const char* fh_last_error(void) { return g_last_error; }

float fh_scale_from_amax(float amax) {
  if (!(amax >= 0.0f) || isinf(amax)) return NAN;
  if (amax == 0.0f) return 1.0f;
  const double target = (double)amax;
  // Start from the nearest FP32 to amax / 2688, then move to the smallest FP32
  // whose product with 2688 (exact in FP64) still covers amax.
  float s = (float)(target / 2688.0);
  while ((double)s * 2688.0 < target) s = nextafterf(s, INFINITY);
  for (;;) {
    const float below = nextafterf(s, 0.0f);
    if (below <= 0.0f || (double)below * 2688.0 < target) break;
    s = below;
  }
  return s;
}

size_t fh_scales_bytes(int64_t rows, int64_t K, int layout) {
  if (rows < 0 || K <= 0 || K % 16 != 0) return 0;
  if (layout == FH_SCALES_ROWMAJOR) return (size_t)rows * (size_t)(K / 16);
  if (layout == FH_SCALES_MMA_TILED) {
    if (K % 64 != 0) return 0;
    return (size_t)((rows + 127) / 128) * 128 * (size_t)(K / 16);
  }
  return 0;
}

int fh_amax(const uint16_t* x_dev, int64_t rows, int64_t cols, int64_t ldx, float* amax_dev,
            fh_stream_t stream) {
  g_last_error[0] = 0;
  if (rows < 0 || cols < 0 || ldx < cols)
    return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_amax: need rows, cols >= 0 and ldx >= cols%s");
  if (amax_dev == nullptr || (x_dev == nullptr && rows * cols > 0))
    return fail(FH_ERR_INVALID_ARG, "fh_amax: null pointer%s");
  if (rows == 0 || cols == 0) return FH_OK;
  if (int st = check_device()) return st;
  cudaError_t e = fh::launch_amax(x_dev, rows, cols, ldx, amax_dev, (cudaStream_t)stream);
  return e == cudaSuccess ? FH_OK : cuda_fail(e, "fh_amax launch");
}

int fh_quantize_act(const uint16_t* x_dev, int64_t M, int64_t K, int64_t ldx, float global_scale,
                    uint8_t* codes_dev, uint8_t* scales_dev, unsigned long long* clip_count_dev,
                    int scale_layout, fh_stream_t stream) {
  g_last_error[0] = 0;
  if (scale_layout != FH_SCALES_ROWMAJOR && scale_layout != FH_SCALES_MMA_TILED)
    return fail(FH_ERR_INVALID_ARG, "fh_quantize_act: unknown scale layout%s");
  if (!(global_scale > 0.0f) || isinf(global_scale))
    return fail(FH_ERR_INVALID_ARG, "fh_quantize_act: global scale must be finite and > 0%s");
  if (M < 0 || K <= 0 || K % 16 != 0 || ldx < K || ldx % 8 != 0)
    return fail(FH_ERR_UNSUPPORTED_SHAPE,
                "fh_quantize_act: need M >= 0, K > 0, K %% 16 == 0, ldx >= K, ldx %% 8 == 0%s");
  if (scale_layout == FH_SCALES_MMA_TILED && K % 64 != 0)
    return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_quantize_act: the tensor-core scale layout needs K %% 64 == 0%s");
  if (M == 0) return FH_OK;
  if (x_dev == nullptr || codes_dev == nullptr || scales_dev == nullptr)
    return fail(FH_ERR_INVALID_ARG, "fh_quantize_act: null pointer%s");
  if (!aligned16(x_dev) || !aligned16(codes_dev) || !aligned16(scales_dev))
    return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_quantize_act: x, codes and scales must be 16-byte aligned%s");
  if (M * (K / 16) > ((int64_t)1 << 40))
    return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_quantize_act: tensor too large%s");
  if (int st = check_device()) return st;
  cudaError_t e = fh::launch_quantize(x_dev, M, K, ldx, global_scale, codes_dev, scales_dev, clip_count_dev,
                                      scale_layout, false, (cudaStream_t)stream);
  return e == cudaSuccess ? FH_OK : cuda_fail(e, "fh_quantize_act launch");
}

int fh_gelu_quantize_act(const uint16_t* x_dev, int64_t M, int64_t K, int64_t ldx, float global_scale,
                         uint8_t* codes_dev, uint8_t* scales_dev, unsigned long long* clip_count_dev,
                         fh_stream_t stream) {
  g_last_error[0] = 0;
  if (!(global_scale > 0.0f) || isinf(global_scale))
    return fail(FH_ERR_INVALID_ARG, "fh_gelu_quantize_act: global scale must be finite and > 0%s");
  if (M < 0 || K <= 0 || K % 64 != 0 || ldx < K || ldx % 8 != 0)
    return fail(FH_ERR_UNSUPPORTED_SHAPE,
                "fh_gelu_quantize_act: need M >= 0, K > 0, K %% 64 == 0, ldx >= K, ldx %% 8 == 0%s");
  if (M == 0) return FH_OK;
  if (x_dev == nullptr || codes_dev == nullptr || scales_dev == nullptr)
    return fail(FH_ERR_INVALID_ARG, "fh_gelu_quantize_act: null pointer%s");
  if (!aligned16(x_dev) || !aligned16(codes_dev) || !aligned16(scales_dev))
    return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_gelu_quantize_act: x, codes and scales must be 16-byte aligned%s");
  if (M * (K / 16) > ((int64_t)1 << 40))
    return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_gelu_quantize_act: tensor too large%s");
  if (int st = check_device()) return st;
  cudaError_t e = fh::launch_quantize(x_dev, M, K, ldx, global_scale, codes_dev, scales_dev, clip_count_dev,
                                      FH_SCALES_MMA_TILED, true, (cudaStream_t)stream);
  return e == cudaSuccess ? FH_OK : cuda_fail(e, "fh_gelu_quantize_act launch");
}

int fh_nvfp4_linear(const uint8_t* a_codes_dev, const uint8_t* a_scales_dev, float a_gscale,
                    const uint8_t* w_codes_dev, const uint8_t* w_scales_dev, float w_gscale,
                    const uint16_t* bias_dev, uint16_t* y_dev, int64_t M, int64_t N, int64_t K,
                    fh_stream_t stream) {
  g_last_error[0] = 0;
  if (!(a_gscale > 0.0f) || isinf(a_gscale) || !(w_gscale > 0.0f) || isinf(w_gscale))
    return fail(FH_ERR_INVALID_ARG, "fh_nvfp4_linear: global scales must be finite and > 0%s");
  if (M < 0 || N < 0 || K <= 0 || K % 64 != 0 || N % 8 != 0)
    return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_nvfp4_linear: need M, N >= 0, K > 0, K %% 64 == 0, N %% 8 == 0%s");
  if (M > 0x7FFFFFFF || N > 0x7FFFFFFF || K > 0x7FFFFFFF)
    return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_nvfp4_linear: each dimension must fit in 31 bits%s");
  if (M == 0 || N == 0) return FH_OK;
  if (a_codes_dev == nullptr || a_scales_dev == nullptr || w_codes_dev == nullptr || w_scales_dev == nullptr ||
      y_dev == nullptr)
    return fail(FH_ERR_INVALID_ARG, "fh_nvfp4_linear: null pointer%s");
  if (!aligned16(a_codes_dev) || !aligned16(a_scales_dev) || !aligned16(w_codes_dev) ||
      !aligned16(w_scales_dev) || !aligned16(y_dev) || (bias_dev != nullptr && !aligned16(bias_dev)))
    return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_nvfp4_linear: every pointer must be 16-byte aligned%s");
  if (int st = check_device()) return st;
  const char* why = nullptr;
  cudaError_t e = fh::launch_nvfp4_linear(a_codes_dev, a_scales_dev, a_gscale, w_codes_dev, w_scales_dev,
                                          w_gscale, bias_dev, y_dev, M, N, K, (cudaStream_t)stream, &why);
  if (e == cudaErrorNotSupported && why != nullptr) return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_nvfp4_linear: %s", why);
  return e == cudaSuccess ? FH_OK : cuda_fail(e, "fh_nvfp4_linear launch");
}

int fh_nvfp4_linear_gelu_quant(const uint8_t* a_codes_dev, const uint8_t* a_scales_dev, float a_gscale,
                               const uint8_t* w_codes_dev, const uint8_t* w_scales_dev, float w_gscale,
                               const uint16_t* bias_dev, float out_gscale, uint8_t* out_codes_dev,
                               uint8_t* out_scales_dev, unsigned long long* out_clip_count_dev,
                               int64_t M, int64_t N, int64_t K, fh_stream_t stream) {
  g_last_error[0] = 0;
  if (!(a_gscale > 0.0f) || isinf(a_gscale) || !(w_gscale > 0.0f) || isinf(w_gscale) || !(out_gscale > 0.0f) ||
      isinf(out_gscale))
    return fail(FH_ERR_INVALID_ARG, "fh_nvfp4_linear_gelu_quant: global scales must be finite and > 0%s");
  if (M < 0 || N < 0 || K <= 0 || K % 64 != 0 || N % 64 != 0)
    return fail(FH_ERR_UNSUPPORTED_SHAPE,
                "fh_nvfp4_linear_gelu_quant: need M, N >= 0, K > 0, K %% 64 == 0, N %% 64 == 0%s");
  if (M > 0x7FFFFFFF || N > 0x7FFFFFFF || K > 0x7FFFFFFF)
    return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_nvfp4_linear_gelu_quant: each dimension must fit in 31 bits%s");
  if (M == 0 || N == 0) return FH_OK;
  if (a_codes_dev == nullptr || a_scales_dev == nullptr || w_codes_dev == nullptr || w_scales_dev == nullptr ||
      out_codes_dev == nullptr || out_scales_dev == nullptr)
    return fail(FH_ERR_INVALID_ARG, "fh_nvfp4_linear_gelu_quant: null pointer%s");
  if (!aligned16(a_codes_dev) || !aligned16(a_scales_dev) || !aligned16(w_codes_dev) || !aligned16(w_scales_dev) ||
      !aligned16(out_codes_dev) || !aligned16(out_scales_dev) || (bias_dev != nullptr && !aligned16(bias_dev)))
    return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_nvfp4_linear_gelu_quant: every pointer must be 16-byte aligned%s");
  if (int st = check_device()) return st;
  const char* why = nullptr;
  cudaError_t e = fh::launch_nvfp4_linear_gelu_quant(a_codes_dev, a_scales_dev, a_gscale, w_codes_dev, w_scales_dev,
                                                     w_gscale, bias_dev, out_gscale, out_codes_dev, out_scales_dev,
                                                     out_clip_count_dev, M, N, K, (cudaStream_t)stream, &why);
  if (e == cudaErrorNotSupported && why != nullptr)
    return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_nvfp4_linear_gelu_quant: %s", why);
  return e == cudaSuccess ? FH_OK : cuda_fail(e, "fh_nvfp4_linear_gelu_quant launch");
}

size_t fh_nvfp4_linear_fused_quant_sync_bytes(int64_t M) {
  if (M < 0 || M > 0x7FFFFFFF) return 0;
  return (size_t)((M + 127) / 128 + 1) * sizeof(uint32_t);
}

int fh_nvfp4_linear_fused_quant(const uint16_t* x_dev, int64_t M, int64_t K, int64_t ldx, float a_gscale,
                                const uint8_t* w_codes_dev, const uint8_t* w_scales_dev, float w_gscale,
                                const uint16_t* bias_dev, uint16_t* y_dev, int64_t N, uint8_t* a_codes_dev,
                                uint8_t* a_scales_dev, unsigned long long* clip_count_dev, uint32_t* sync_dev,
                                fh_stream_t stream) {
  g_last_error[0] = 0;
  if (!(a_gscale > 0.0f) || isinf(a_gscale) || !(w_gscale > 0.0f) || isinf(w_gscale))
    return fail(FH_ERR_INVALID_ARG, "fh_nvfp4_linear_fused_quant: global scales must be finite and > 0%s");
  if (M < 0 || N < 0 || K <= 0 || K % 64 != 0 || N % 8 != 0 || ldx < K || ldx % 8 != 0)
    return fail(FH_ERR_UNSUPPORTED_SHAPE,
                "fh_nvfp4_linear_fused_quant: need M, N >= 0, K > 0, K %% 64 == 0, N %% 8 == 0, ldx >= K, "
                "ldx %% 8 == 0%s");
  if (M > 0x7FFFFFFF || N > 0x7FFFFFFF || K > 0x7FFFFFFF || ((M + 127) / 128) * (K / 16) > 0x7FFFFFFF)
    return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_nvfp4_linear_fused_quant: tensor too large%s");
  if (M == 0 || N == 0) return FH_OK;
  if (x_dev == nullptr || w_codes_dev == nullptr || w_scales_dev == nullptr || y_dev == nullptr ||
      a_codes_dev == nullptr || a_scales_dev == nullptr || sync_dev == nullptr)
    return fail(FH_ERR_INVALID_ARG, "fh_nvfp4_linear_fused_quant: null pointer%s");
  if (!aligned16(x_dev) || !aligned16(w_codes_dev) || !aligned16(w_scales_dev) || !aligned16(y_dev) ||
      !aligned16(a_codes_dev) || !aligned16(a_scales_dev) || (bias_dev != nullptr && !aligned16(bias_dev)) ||
      (reinterpret_cast<uintptr_t>(sync_dev) & 3u) != 0)
    return fail(FH_ERR_UNSUPPORTED_SHAPE,
                "fh_nvfp4_linear_fused_quant: sync must be 4-byte aligned, every other pointer 16-byte aligned%s");
  if (int st = check_device()) return st;
  const char* why = nullptr;
  cudaError_t e = fh::launch_nvfp4_linear_quant_prologue(x_dev, ldx, a_gscale, w_codes_dev, w_scales_dev, w_gscale,
                                                         bias_dev, y_dev, a_codes_dev, a_scales_dev, clip_count_dev,
                                                         sync_dev, M, N, K, (cudaStream_t)stream, &why);
  if (e == cudaErrorNotSupported && why != nullptr)
    return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_nvfp4_linear_fused_quant: %s", why);
  return e == cudaSuccess ? FH_OK : cuda_fail(e, "fh_nvfp4_linear_fused_quant launch");
}

size_t fh_nvfp4_linear_host_workspace_bytes(int64_t K, int64_t N, int64_t chunk_rows) {
  if (K <= 0 || K % 64 != 0 || N <= 0 || N % 8 != 0 || chunk_rows <= 0 || chunk_rows % 128 != 0 ||
      K > 0x7FFFFFFF || N > 0x7FFFFFFF || chunk_rows > 0x7FFFFFFF)
    return 0;
  return fh::host_linear_workspace_bytes(K, N, chunk_rows);
}

int fh_nvfp4_linear_host(const uint16_t* x_host, int64_t M, int64_t K, float a_gscale, const uint8_t* w_codes_dev,
                         const uint8_t* w_scales_dev, float w_gscale, const uint16_t* bias_dev, int64_t N,
                         uint16_t* y_host, unsigned long long* clip_count_dev, int64_t chunk_rows,
                         void* workspace_dev, size_t workspace_bytes, fh_stream_t stream) {
  g_last_error[0] = 0;
  if (!(a_gscale > 0.0f) || isinf(a_gscale) || !(w_gscale > 0.0f) || isinf(w_gscale))
    return fail(FH_ERR_INVALID_ARG, "fh_nvfp4_linear_host: global scales must be finite and > 0%s");
  if (M < 0 || M > 0x7FFFFFFF)
    return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_nvfp4_linear_host: need 0 <= M < 2^31%s");
  const size_t need = fh_nvfp4_linear_host_workspace_bytes(K, N, chunk_rows);
  if (need == 0)
    return fail(FH_ERR_UNSUPPORTED_SHAPE,
                "fh_nvfp4_linear_host: need K > 0, K %% 64 == 0, N > 0, N %% 8 == 0, chunk_rows > 0, "
                "chunk_rows %% 128 == 0%s");
  if (M == 0) return FH_OK;
  if (x_host == nullptr || y_host == nullptr || w_codes_dev == nullptr || w_scales_dev == nullptr ||
      workspace_dev == nullptr)
    return fail(FH_ERR_INVALID_ARG, "fh_nvfp4_linear_host: null pointer%s");
  if (workspace_bytes < need)
    return fail(FH_ERR_INVALID_ARG, "fh_nvfp4_linear_host: workspace smaller than "
                                    "fh_nvfp4_linear_host_workspace_bytes(K, N, chunk_rows)%s");
  if ((reinterpret_cast<uintptr_t>(workspace_dev) & 255u) != 0 || !aligned16(w_codes_dev) ||
      !aligned16(w_scales_dev) || (bias_dev != nullptr && !aligned16(bias_dev)))
    return fail(FH_ERR_UNSUPPORTED_SHAPE,
                "fh_nvfp4_linear_host: workspace must be 256-byte aligned, weights and bias 16-byte aligned%s");
  if (int st = check_device()) return st;
  const char* why = nullptr;
  cudaError_t e = fh::launch_nvfp4_linear_host(x_host, M, K, a_gscale, w_codes_dev, w_scales_dev, w_gscale, bias_dev,
                                               N, y_host, clip_count_dev, chunk_rows, workspace_dev,
                                               (cudaStream_t)stream, &why);
  if (e == cudaErrorNotSupported && why != nullptr)
    return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_nvfp4_linear_host: %s", why);
  return e == cudaSuccess ? FH_OK : cuda_fail(e, "fh_nvfp4_linear_host");
}

int fh_nvfp4_linear_host_noalloc(const uint16_t* x_host, int64_t M, int64_t K, float a_gscale,
                                 const uint8_t* w_codes_dev, const uint8_t* w_scales_dev, float w_gscale,
                                 const uint16_t* bias_dev, int64_t N, uint16_t* y_host,
                                 unsigned long long* clip_count_dev, fh_stream_t stream) {
  g_last_error[0] = 0;
  if (!(a_gscale > 0.0f) || isinf(a_gscale) || !(w_gscale > 0.0f) || isinf(w_gscale))
    return fail(FH_ERR_INVALID_ARG, "fh_nvfp4_linear_host_noalloc: global scales must be finite and > 0%s");
  if (M < 0 || M > 0x7FFFFFFF || K <= 0 || K % 64 != 0 || N <= 0 || N % 8 != 0 || K > 0x7FFFFFFF ||
      N > 0x7FFFFFFF)
    return fail(FH_ERR_UNSUPPORTED_SHAPE,
                "fh_nvfp4_linear_host_noalloc: need 0 <= M < 2^31, K > 0, K %% 64 == 0, N > 0, N %% 8 == 0%s");
  if (fh::noalloc_chunk_rows(K, N) == 0) {
    char msg[200];
    snprintf(msg, sizeof msg, "one 128-row chunk needs %zu bytes of scratch, more than the library's static %u",
             fh::noalloc_chunk_bytes(K, N, 128), (unsigned)FH_NOALLOC_SCRATCH_BYTES);
    return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_nvfp4_linear_host_noalloc: %s", msg);
  }
  if (M == 0) return FH_OK;
  if (x_host == nullptr || y_host == nullptr || w_codes_dev == nullptr || w_scales_dev == nullptr)
    return fail(FH_ERR_INVALID_ARG, "fh_nvfp4_linear_host_noalloc: null pointer%s");
  if (!aligned16(w_codes_dev) || !aligned16(w_scales_dev) || (bias_dev != nullptr && !aligned16(bias_dev)))
    return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_nvfp4_linear_host_noalloc: weights and bias must be 16-byte aligned%s");
  if (int st = check_device()) return st;
  const char* why = nullptr;
  cudaError_t e = fh::launch_nvfp4_linear_host_noalloc(x_host, M, K, a_gscale, w_codes_dev, w_scales_dev, w_gscale,
                                                       bias_dev, N, y_host, clip_count_dev, (cudaStream_t)stream, &why);
  if (e == cudaErrorNotSupported && why != nullptr)
    return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_nvfp4_linear_host_noalloc: %s", why);
  return e == cudaSuccess ? FH_OK : cuda_fail(e, "fh_nvfp4_linear_host_noalloc");
}

int fh_scales_to_rowmajor(const uint8_t* tiled_dev, uint8_t* rowmajor_dev, int64_t rows, int64_t K,
                          fh_stream_t stream) {
  g_last_error[0] = 0;
  if (rows < 0 || K <= 0 || K % 64 != 0)
    return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_scales_to_rowmajor: need rows >= 0, K > 0, K %% 64 == 0%s");
  if (rows == 0) return FH_OK;
  if (tiled_dev == nullptr || rowmajor_dev == nullptr)
    return fail(FH_ERR_INVALID_ARG, "fh_scales_to_rowmajor: null pointer%s");
  if (int st = check_device()) return st;
  cudaError_t e = fh::launch_scales_to_rowmajor(tiled_dev, rowmajor_dev, rows, K, (cudaStream_t)stream);
  return e == cudaSuccess ? FH_OK : cuda_fail(e, "fh_scales_to_rowmajor launch");
}

int fh_gelu_bf16(const uint16_t* x_dev, uint16_t* y_dev, int64_t n, fh_stream_t stream) {
  g_last_error[0] = 0;
  if (n < 0) return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_gelu_bf16: n must be >= 0%s");
  if (n == 0) return FH_OK;
  if (x_dev == nullptr || y_dev == nullptr) return fail(FH_ERR_INVALID_ARG, "fh_gelu_bf16: null pointer%s");
  if (!aligned16(x_dev) || !aligned16(y_dev))
    return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_gelu_bf16: x and y must be 16-byte aligned%s");
  if (int st = check_device()) return st;
  cudaError_t e = fh::launch_gelu(x_dev, y_dev, n, (cudaStream_t)stream);
  return e == cudaSuccess ? FH_OK : cuda_fail(e, "fh_gelu_bf16 launch");
}

int fh_quantize_int8_rows(const uint16_t* x_dev, int64_t rows, int64_t d, int64_t ldx, int8_t* q_dev,
                          float* scales_dev, fh_stream_t stream) {
  g_last_error[0] = 0;
  if (rows < 0 || d <= 0 || d % 8 != 0 || ldx < d || ldx % 8 != 0)
    return fail(FH_ERR_UNSUPPORTED_SHAPE,
                "fh_quantize_int8_rows: need rows >= 0, d > 0, d %% 8 == 0, ldx >= d, ldx %% 8 == 0%s");
  if (rows == 0) return FH_OK;
  if (x_dev == nullptr || q_dev == nullptr || scales_dev == nullptr)
    return fail(FH_ERR_INVALID_ARG, "fh_quantize_int8_rows: null pointer%s");
  if (!aligned16(x_dev) || !aligned16(q_dev) || (reinterpret_cast<uintptr_t>(scales_dev) & 3u) != 0)
    return fail(FH_ERR_UNSUPPORTED_SHAPE,
                "fh_quantize_int8_rows: x and q must be 16-byte aligned, scales 4-byte aligned%s");
  if (int st = check_device()) return st;
  cudaError_t e = fh::launch_int8_quantize_rows(x_dev, rows, d, ldx, q_dev, scales_dev, (cudaStream_t)stream);
  return e == cudaSuccess ? FH_OK : cuda_fail(e, "fh_quantize_int8_rows launch");
}

int fh_int8_attention_scores(const int8_t* q_dev, const float* q_scales_dev, const int8_t* k_dev,
                             const float* k_scales_dev, float sm_scale, float* s_dev, int64_t heads, int64_t tq,
                             int64_t tk, int64_t d, fh_stream_t stream) {
  g_last_error[0] = 0;
  if (!isfinite(sm_scale))
    return fail(FH_ERR_INVALID_ARG, "fh_int8_attention_scores: sm_scale must be finite%s");
  if (heads < 0 || tq < 0 || tk < 0 || d <= 0 || d % 16 != 0)
    return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_int8_attention_scores: need heads, tq, tk >= 0, d > 0, d %% 16 == 0%s");
  if (heads > 0x7FFFFFFF || tq > 0x7FFFFFFF || tk > 0x7FFFFFFF || d > 65536)
    return fail(FH_ERR_UNSUPPORTED_SHAPE,
                "fh_int8_attention_scores: heads, tq, tk must fit in 31 bits and d <= 65536%s");
  if (heads == 0 || tq == 0 || tk == 0) return FH_OK;
  if (heads * ((tq + 127) / 128) * ((tk + 255) / 256) > 0x7FFFFFFF || tq * tk * 4 >= ((int64_t)1 << 40) ||
      tq * d >= ((int64_t)1 << 40) || tk * d >= ((int64_t)1 << 40))
    return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_int8_attention_scores: tensor too large%s");
  if (q_dev == nullptr || q_scales_dev == nullptr || k_dev == nullptr || k_scales_dev == nullptr ||
      s_dev == nullptr)
    return fail(FH_ERR_INVALID_ARG, "fh_int8_attention_scores: null pointer%s");
  if (!aligned16(q_dev) || !aligned16(k_dev) || !aligned16(s_dev))
    return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_int8_attention_scores: q, k and s must be 16-byte aligned%s");
  if (int st = check_device()) return st;
  const char* why = nullptr;
  cudaError_t e = fh::launch_int8_scores(q_dev, q_scales_dev, k_dev, k_scales_dev, sm_scale, s_dev, heads, tq, tk,
                                         d, (cudaStream_t)stream, &why);
  if (e == cudaErrorNotSupported && why != nullptr)
    return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_int8_attention_scores: %s", why);
  return e == cudaSuccess ? FH_OK : cuda_fail(e, "fh_int8_attention_scores launch");
}

int fh_adaln_modulation(const uint16_t* temb_dev, int64_t bt, int64_t d, const uint16_t* basis_dev, int64_t r,
                        const uint16_t* proj_dev, const uint16_t* bias_dev, int64_t blocks, int64_t n,
                        float* code_dev, float* mod_dev, fh_stream_t stream) {
  g_last_error[0] = 0;
  if (bt < 0 || d <= 0 || d % 8 != 0 || blocks < 0 || n < 0)
    return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_adaln_modulation: need bt, blocks, n >= 0, d > 0, d %% 8 == 0%s");
  if (r != 8 && r != 16 && r != 24 && r != 32)
    return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_adaln_modulation: the basis rank r must be 8, 16, 24 or 32%s");
  if (blocks * n > 0x7FFFFFFF || bt > 0x7FFFFFFF || d > ((int64_t)1 << 40))
    return fail(FH_ERR_UNSUPPORTED_SHAPE, "fh_adaln_modulation: tensor too large%s");
  if (bt == 0) return FH_OK;
  if (temb_dev == nullptr || basis_dev == nullptr || code_dev == nullptr ||
      (blocks * n > 0 && (proj_dev == nullptr || mod_dev == nullptr)))
    return fail(FH_ERR_INVALID_ARG, "fh_adaln_modulation: null pointer%s");
  if (!aligned16(temb_dev) || !aligned16(basis_dev) || (proj_dev != nullptr && !aligned16(proj_dev)) ||
      (reinterpret_cast<uintptr_t>(bias_dev) & 1u) != 0 || (reinterpret_cast<uintptr_t>(code_dev) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(mod_dev) & 3u) != 0)
    return fail(FH_ERR_UNSUPPORTED_SHAPE,
                "fh_adaln_modulation: temb, basis and proj must be 16-byte aligned, bias 2-byte, code and mod "
                "4-byte%s");
  if (int st = check_device()) return st;
  cudaError_t e = fh::launch_adaln_modulation(temb_dev, bt, d, basis_dev, r, proj_dev, bias_dev, blocks, n, code_dev,
                                              mod_dev, (cudaStream_t)stream);
  return e == cudaSuccess ? FH_OK : cuda_fail(e, "fh_adaln_modulation launch");
}

int fh_selftest_bounded_wait(uint32_t limit_us, fh_stream_t stream) {
  g_last_error[0] = 0;
  if (limit_us == 0 || limit_us > 2000000u)
    return fail(FH_ERR_INVALID_ARG, "fh_selftest_bounded_wait: limit must be 1 us .. 2 s%s");
  if (int st = check_device()) return st;
  cudaError_t e = fh::launch_bounded_wait_selftest((uint64_t)limit_us * 1000u, (cudaStream_t)stream);
  return e == cudaSuccess ? FH_OK : cuda_fail(e, "fh_selftest_bounded_wait launch");
}

int fh_selftest_mma_rate(int32_t iters, int32_t with_scale_copies, int32_t* pairs_out, fh_stream_t stream) {
  g_last_error[0] = 0;
  if (iters < 1 || iters > 1000000 || pairs_out == nullptr)
    return fail(FH_ERR_INVALID_ARG, "fh_selftest_mma_rate: need 1 <= iters <= 1e6 and pairs_out%s");
  if (int st = check_device()) return st;
  int pairs = 0;
  cudaError_t e = fh::launch_mma_rate_probe((int)iters, with_scale_copies ? 1 : 0, &pairs, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "fh_selftest_mma_rate launch");
  *pairs_out = pairs;
  return FH_OK;
}

int fh_device_status(fh_stream_t stream) {
  g_last_error[0] = 0;
  if (int st = check_device()) return st;
  unsigned int bits = 0, qbits = 0, ibits = 0;
  cudaError_t e = fh::read_and_clear_device_error(&bits, (cudaStream_t)stream);
  if (e == cudaSuccess) e = fh::read_and_clear_quant_error(&qbits);
  if (e == cudaSuccess) e = fh::read_and_clear_int8_error(&ibits);
  if (e != cudaSuccess) return cuda_fail(e, "fh_device_status");
  bits |= qbits | ibits;
  if (bits & fh::kDevErrTimeout)
    return fail(FH_ERR_TIMEOUT, "a kernel gave up on a bounded on-chip wait%s");
  return FH_OK;
}

}  // extern "C"
