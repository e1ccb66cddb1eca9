// fh_host.cu -- the layer on host buffers: BF16 activations in page-locked host
// memory in, BF16 outputs back to host memory, pipelined over row chunks so that
// the PCIe transfers in both directions and the GPU work overlap.
//
// Per chunk c (chunk_rows rows of x):
//   caller's stream S:  H2D x[c] -> x slot c%2;  quantize -> codes/scales;
//                       wait until D2H of chunk c-2 has read y slot c%2;
//                       GEMM -> y slot c%2;  record done[c%2]
//   copy stream D:      wait done[c%2];  D2H y slot c%2 -> y_host[c];
//                       record read[c%2]
// and at the end S waits for the last D2H, so the call is ordered on S like any
// other: work enqueued on S afterwards sees y_host complete.  The download
// (N/K times the upload) overlaps the next chunks' uploads and kernels.
// The device workspace is the caller's; the library allocates no memory.  The
// copy stream and four events are created once per host thread and device.
#include <cuda_runtime.h>
#include <stdint.h>

#include "fh_internal.h"

namespace fh {

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

struct Workspace {
  size_t x_slot, codes, scales, y_slot, total;
};

Workspace workspace_layout(int64_t K, int64_t N, int64_t chunk_rows) {
  Workspace w;
  w.x_slot = align_up((size_t)chunk_rows * (size_t)K * 2);
  w.codes = align_up((size_t)chunk_rows * (size_t)K / 2);
  w.scales = align_up((size_t)((chunk_rows + 127) / 128) * 128 * (size_t)(K / 16));
  w.y_slot = align_up((size_t)chunk_rows * (size_t)N * 2);
  w.total = 2 * w.x_slot + w.codes + w.scales + 2 * w.y_slot;
  return w;
}

struct CopyEngine {
  int device = -1;
  cudaStream_t d2h = nullptr;
  cudaEvent_t done[2] = {nullptr, nullptr};  // GEMM of the slot's chunk finished
  cudaEvent_t read[2] = {nullptr, nullptr};  // D2H of the slot's chunk finished
};

cudaError_t copy_engine(CopyEngine** out) {
  thread_local CopyEngine eng;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (eng.device != dev) {
    // A new device for this thread: earlier objects belong to another device
    // and are left alone.
    CopyEngine fresh;
    e = cudaStreamCreateWithFlags(&fresh.d2h, cudaStreamNonBlocking);
    for (int i = 0; i < 2 && e == cudaSuccess; ++i) {
      e = cudaEventCreateWithFlags(&fresh.done[i], cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&fresh.read[i], cudaEventDisableTiming);
    }
    if (e != cudaSuccess) return e;
    fresh.device = dev;
    eng = fresh;
  }
  *out = &eng;
  return cudaSuccess;
}

}  // namespace

size_t host_linear_workspace_bytes(int64_t K, int64_t N, int64_t chunk_rows) {
  return workspace_layout(K, N, chunk_rows).total;
}

cudaError_t launch_nvfp4_linear_host(const uint16_t* x_host, int64_t M, int64_t K, float a_g, const uint8_t* w_codes,
                                     const uint8_t* w_scales, float w_g, const uint16_t* bias, int64_t N,
                                     uint16_t* y_host, unsigned long long* clip, int64_t chunk_rows, void* workspace,
                                     cudaStream_t s, const char** why) {
  CopyEngine* eng = nullptr;
  cudaError_t e = copy_engine(&eng);
  if (e != cudaSuccess) return e;
  const Workspace L = workspace_layout(K, N, chunk_rows);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  uint16_t* x_slot[2] = {reinterpret_cast<uint16_t*>(base), reinterpret_cast<uint16_t*>(base + L.x_slot)};
  uint8_t* codes = base + 2 * L.x_slot;
  uint8_t* scales = codes + L.codes;
  uint16_t* y_slot[2] = {reinterpret_cast<uint16_t*>(scales + L.scales),
                         reinterpret_cast<uint16_t*>(scales + L.scales + L.y_slot)};
  const int64_t chunks = (M + chunk_rows - 1) / chunk_rows;
  for (int64_t c = 0; c < chunks; ++c) {
    const int slot = (int)(c & 1);
    const int64_t r0 = c * chunk_rows;
    const int64_t rows = M - r0 < chunk_rows ? M - r0 : chunk_rows;
    e = cudaMemcpyAsync(x_slot[slot], x_host + r0 * K, (size_t)rows * (size_t)K * 2, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return e;
    e = launch_quantize(x_slot[slot], rows, K, K, a_g, codes, scales, clip, FH_SCALES_MMA_TILED, false, s);
    if (e != cudaSuccess) return e;
    e = cudaStreamWaitEvent(s, eng->read[slot], 0);  // the slot's previous download has read it
    if (e != cudaSuccess) return e;
    e = launch_nvfp4_linear(codes, scales, a_g, w_codes, w_scales, w_g, bias, y_slot[slot], rows, N, K, s, why);
    if (e != cudaSuccess) return e;
    e = cudaEventRecord(eng->done[slot], s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(eng->d2h, eng->done[slot], 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(y_host + r0 * N, y_slot[slot], (size_t)rows * (size_t)N * 2, cudaMemcpyDeviceToHost,
                          eng->d2h);
    if (e == cudaSuccess) e = cudaEventRecord(eng->read[slot], eng->d2h);
    if (e != cudaSuccess) return e;
  }
  // The call completes on the caller's stream once the last download has landed.
  return cudaStreamWaitEvent(s, eng->read[(chunks - 1) & 1], 0);
}

}  // namespace fh
