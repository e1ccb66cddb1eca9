// fh_host.cu -- the layer on host buffers: BF16 activations in page-locked host
// memory in, BF16 outputs back to host memory, pipelined over row chunks so that
// the uploads, the kernels and the downloads overlap.
//
// Three streams take part: the caller's stream S runs the kernels, and two copy
// streams the library keeps per host thread and device run the transfers, U the
// uploads and D the downloads.  The device workspace holds two x slots, one set
// of codes and scales, and two y slots.  Per chunk c (slot c % 2):
//   U:  [c >= 2: wait x_free[slot]]  H2D x[c] -> x slot;  record x_ready[slot]
//   S:  wait x_ready[slot];  quantize -> codes/scales;  record x_free[slot];
//       [c >= 2: wait y_free[slot]]  GEMM -> y slot;  record y_done[slot]
//   D:  wait y_done[slot];  D2H y slot -> y_host[c];  record y_free[slot]
// so the upload of chunk c + 1 runs under the kernels of chunk c, and the
// download of chunk c under the kernels of chunk c + 1.  U and D first wait for
// the work enqueued on S before the call, and at the end (also after a failed
// step) S waits for everything U and D were given, so the call is ordered on S
// like any other: work enqueued on S afterwards sees y_host complete.
// The device workspace is the caller's; the library allocates no memory.  The
// two copy streams and eleven events are created once per host thread and device.
#include <cuda_runtime.h>
#include <stdint.h>

#include "fh_internal.h"

namespace fh {

namespace {

constexpr size_t kAlign = 256;
constexpr int kMaxDevices = 64;

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
  bool ready = false;
  cudaStream_t up = nullptr, down = nullptr;
  cudaEvent_t entry = nullptr;                      // S reached the call
  cudaEvent_t x_ready[2] = {nullptr, nullptr};      // upload of the slot's chunk landed
  cudaEvent_t x_free[2] = {nullptr, nullptr};       // quantizer of the slot's chunk read it
  cudaEvent_t y_done[2] = {nullptr, nullptr};       // GEMM of the slot's chunk finished
  cudaEvent_t y_free[2] = {nullptr, nullptr};       // download of the slot's chunk read it
  cudaEvent_t up_joined = nullptr, down_joined = nullptr;
};

cudaError_t create_engine(CopyEngine* g) {
  cudaError_t e = cudaStreamCreateWithFlags(&g->up, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&g->down, cudaStreamNonBlocking);
  cudaEvent_t* ev[] = {&g->entry,     &g->x_ready[0], &g->x_ready[1], &g->x_free[0],   &g->x_free[1],
                       &g->y_done[0], &g->y_done[1],  &g->y_free[0],  &g->y_free[1], &g->up_joined,
                       &g->down_joined};
  for (cudaEvent_t* p : ev)
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(p, cudaEventDisableTiming);
  if (e != cudaSuccess) {
    // Leave nothing half-built behind: destroy what was created.
    for (cudaEvent_t* p : ev) {
      if (*p != nullptr) cudaEventDestroy(*p);
      *p = nullptr;
    }
    if (g->up != nullptr) cudaStreamDestroy(g->up);
    if (g->down != nullptr) cudaStreamDestroy(g->down);
    g->up = g->down = nullptr;
    return e;
  }
  g->ready = true;
  return cudaSuccess;
}

// The copy engine of this host thread for the current device, created on first
// use (one per device, so a thread that moves between devices reuses each).
cudaError_t copy_engine(CopyEngine** out) {
  thread_local CopyEngine engines[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  CopyEngine& g = engines[dev];
  if (!g.ready) {
    e = create_engine(&g);
    if (e != cudaSuccess) return e;
  }
  *out = &g;
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
  CopyEngine* g = nullptr;
  cudaError_t e = copy_engine(&g);
  if (e != cudaSuccess) return e;
  const Workspace L = workspace_layout(K, N, chunk_rows);
  uint8_t* base = static_cast<uint8_t*>(workspace);
  uint16_t* x_slot[2] = {reinterpret_cast<uint16_t*>(base), reinterpret_cast<uint16_t*>(base + L.x_slot)};
  uint8_t* codes = base + 2 * L.x_slot;
  uint8_t* scales = codes + L.codes;
  uint16_t* y_slot[2] = {reinterpret_cast<uint16_t*>(scales + L.scales),
                         reinterpret_cast<uint16_t*>(scales + L.scales + L.y_slot)};
  const int64_t chunks = (M + chunk_rows - 1) / chunk_rows;

  // The copy streams start after the work enqueued on S before this call.
  e = cudaEventRecord(g->entry, s);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(g->up, g->entry, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(g->down, g->entry, 0);
  for (int64_t c = 0; c < chunks && e == cudaSuccess; ++c) {
    const int slot = (int)(c & 1);
    const int64_t r0 = c * chunk_rows;
    const int64_t rows = M - r0 < chunk_rows ? M - r0 : chunk_rows;
    // Upload, once the quantizer of chunk c - 2 has read the slot.
    if (c >= 2) e = cudaStreamWaitEvent(g->up, g->x_free[slot], 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(x_slot[slot], x_host + r0 * K, (size_t)rows * (size_t)K * 2, cudaMemcpyHostToDevice,
                          g->up);
    if (e == cudaSuccess) e = cudaEventRecord(g->x_ready[slot], g->up);
    // Kernels on the caller's stream.
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, g->x_ready[slot], 0);
    if (e == cudaSuccess)
      e = launch_quantize(x_slot[slot], rows, K, K, a_g, codes, scales, clip, FH_SCALES_MMA_TILED, false, s);
    if (e == cudaSuccess) e = cudaEventRecord(g->x_free[slot], s);
    if (e == cudaSuccess && c >= 2) e = cudaStreamWaitEvent(s, g->y_free[slot], 0);
    if (e == cudaSuccess)
      e = launch_nvfp4_linear(codes, scales, a_g, w_codes, w_scales, w_g, bias, y_slot[slot], rows, N, K, s, why);
    if (e == cudaSuccess) e = cudaEventRecord(g->y_done[slot], s);
    // Download, once the GEMM has written the slot.
    if (e == cudaSuccess) e = cudaStreamWaitEvent(g->down, g->y_done[slot], 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(y_host + r0 * N, y_slot[slot], (size_t)rows * (size_t)N * 2, cudaMemcpyDeviceToHost,
                          g->down);
    if (e == cudaSuccess) e = cudaEventRecord(g->y_free[slot], g->down);
  }
  // Join both copy streams back into S, also after a failed step, so that
  // nothing this call enqueued is still running once S has passed this point.
  cudaError_t j = cudaEventRecord(g->up_joined, g->up);
  if (j == cudaSuccess) j = cudaStreamWaitEvent(s, g->up_joined, 0);
  if (j == cudaSuccess) j = cudaEventRecord(g->down_joined, g->down);
  if (j == cudaSuccess) j = cudaStreamWaitEvent(s, g->down_joined, 0);
  return e != cudaSuccess ? e : j;
}

}  // namespace fh
