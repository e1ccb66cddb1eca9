// fh_noalloc.cu -- the host-buffer layer for callers that cannot allocate
// device memory.
//
// fh_nvfp4_linear_host stages its row chunks in a device workspace that the
// caller allocates.  Some callers cannot do that: a serving engine or a host
// application that reserves all of the device's memory for its own pool up
// front (so a cudaMalloc fails or fragments that pool), a plugin that may only
// use memory handed to it, or a latency-bound caller that must not pay for
// cudaMalloc / cudaFree, which can synchronize the device.  This variant needs
// no workspace: it stages its chunks in a fixed scratch array in the library's
// own device memory (a file-scope __device__ array, so the CUDA runtime sets
// it aside when it loads this module on a device, and it stays until the
// process exits).  The array holds one chunk of x, its codes and scales, and
// its output; each chunk is uploaded, quantized, multiplied and downloaded in
// order on the caller's stream, so the calls serialize on that stream and
// nothing overlaps inside one call.
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include "fh_internal.h"

namespace fh {

namespace {

constexpr size_t kNoAllocAlign = 256;
static_assert(FH_NOALLOC_SCRATCH_BYTES % kNoAllocAlign == 0, "scratch size");

// The scratch array.  In host code its name stands for a host-side shadow, not
// for the device memory: host code must take the device address with
// cudaGetSymbolAddress and pass that to the copies and kernels.
static __device__ __align__(256) uint8_t g_noalloc_scratch[FH_NOALLOC_SCRATCH_BYTES];

size_t up(size_t v) { return (v + kNoAllocAlign - 1) / kNoAllocAlign * kNoAllocAlign; }

struct ScratchLayout {
  size_t x, codes, scales, y, total;
};

ScratchLayout scratch_layout(int64_t K, int64_t N, int64_t rows) {
  ScratchLayout l;
  l.x = up((size_t)rows * (size_t)K * 2);
  l.codes = up((size_t)rows * (size_t)K / 2);
  l.scales = up((size_t)((rows + 127) / 128) * 128 * (size_t)(K / 16));
  l.y = up((size_t)rows * (size_t)N * 2);
  l.total = l.x + l.codes + l.scales + l.y;
  return l;
}

// Device address of the scratch array on the current device.  The first call
// on a device looks it up (with that device current) and keeps it; later calls
// read the per-device table.
cudaError_t scratch_address(uint8_t** out) {
  static std::atomic<uint8_t*> addr[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  uint8_t* p = (dev >= 0 && dev < kMaxDevices) ? addr[dev].load(std::memory_order_acquire) : nullptr;
  if (p == nullptr) {
    void* q = nullptr;
    e = cudaGetSymbolAddress(&q, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    p = static_cast<uint8_t*>(q);
    if (dev >= 0 && dev < kMaxDevices) addr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return cudaSuccess;
}

}  // namespace

int64_t noalloc_chunk_rows(int64_t K, int64_t N) {
  // Largest multiple of 128 rows whose chunk fits the scratch array.
  const double per_row = 2.0 * (double)K + 0.5 * (double)K + (double)K / 16.0 + 2.0 * (double)N;
  int64_t rows = (int64_t)((double)FH_NOALLOC_SCRATCH_BYTES / per_row) / 128 * 128;
  while (rows >= 128 && scratch_layout(K, N, rows).total > (size_t)FH_NOALLOC_SCRATCH_BYTES) rows -= 128;
  return rows >= 128 ? rows : 0;
}

size_t noalloc_chunk_bytes(int64_t K, int64_t N, int64_t rows) { return scratch_layout(K, N, rows).total; }

cudaError_t launch_nvfp4_linear_host_noalloc(const uint16_t* x_host, int64_t M, int64_t K, float a_g,
                                             const uint8_t* w_codes, const uint8_t* w_scales, float w_g,
                                             const uint16_t* bias, int64_t N, uint16_t* y_host,
                                             unsigned long long* clip, cudaStream_t s, const char** why) {
  const int64_t chunk = noalloc_chunk_rows(K, N);
  uint8_t* base = nullptr;
  cudaError_t e = scratch_address(&base);
  if (e != cudaSuccess) return e;
  const ScratchLayout L = scratch_layout(K, N, chunk);
  uint16_t* xs = reinterpret_cast<uint16_t*>(base);
  uint8_t* codes = base + L.x;
  uint8_t* scales = codes + L.codes;
  uint16_t* ys = reinterpret_cast<uint16_t*>(scales + L.scales);
  // Every byte a chunk reads is written earlier in the same chunk (x by the
  // upload, codes and scales -- padding rows included -- by the quantizer, y
  // by the GEMM), so nothing left in the array by an earlier call is read and
  // nothing needs clearing.
  for (int64_t r0 = 0; r0 < M && e == cudaSuccess; r0 += chunk) {
    const int64_t rows = M - r0 < chunk ? M - r0 : chunk;
    e = cudaMemcpyAsync(xs, x_host + r0 * K, (size_t)rows * (size_t)K * 2, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess)
      e = launch_quantize(xs, rows, K, K, a_g, codes, scales, clip, FH_SCALES_MMA_TILED, false, s);
    if (e == cudaSuccess)
      e = launch_nvfp4_linear(codes, scales, a_g, w_codes, w_scales, w_g, bias, ys, rows, N, K, s, why);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(y_host + r0 * N, ys, (size_t)rows * (size_t)N * 2, cudaMemcpyDeviceToHost, s);
  }
  return e;
}

}  // namespace fh
