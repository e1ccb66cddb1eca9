// fh_adaln.cu -- AdaLN timestep conditioning through a shared low-rank basis.
//
// FastH3 Trim (comfyui-wiki news), "What Trim changes": AdaLN maps the
// 2,688-wide time embedding to six modulation vectors per block; Trim replaces
// the per-block projections with one shared 2,688 -> 16 basis and a small
// projection per block, both stored in FP16.  With BF16 embeddings e [bt, d]:
//   code[b, j]   = sum_k basis[j, k] e[b, k]                       (FP32)
//   mod[l, b, i] = sum_j proj[l, i, j] code[b, j] + bias[l, i]      (FP32)
//
// Two kernels, chained by programmatic dependent launch:
//   adaln_code_kernel  one warp per (b, j): a 16-byte-load dot product over d.
//                      It lets the dependent grid start at once.
//   adaln_mod_kernel   one thread per (l, i): its r FP16 weights and its bias
//                      are loaded into registers before griddepcontrol.wait, so
//                      that the HBM read of the projections overlaps the code
//                      kernel; then the codes are staged in shared memory (128
//                      timesteps at a time) and each timestep's row of
//                      modulations is written with coalesced FP32 stores.
// The work is HBM-bound: the projections are read once, the modulations
// written once.  Neither kernel waits on anything it must bound.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fh_internal.h"

namespace fh {

namespace {

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float2 half2_to_float2(uint32_t w) {
  __half2 h;
  *reinterpret_cast<uint32_t*>(&h) = w;
  return __half22float2(h);
}

// code [bt, r] = e [bt, d] . basis^T, basis [r, d]; d % 8 == 0.
__global__ void __launch_bounds__(256) adaln_code_kernel(const uint16_t* __restrict__ e, int64_t bt, int64_t d,
                                                         const uint16_t* __restrict__ basis, int r,
                                                         float* __restrict__ code) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); w < bt * r; w += warps) {
    const int64_t b = w / r;
    const int j = (int)(w % r);
    const uint16_t* er = e + b * d;
    const uint16_t* br = basis + (int64_t)j * d;
    float acc = 0.0f;
    for (int64_t c = 8 * lane; c < d; c += 256) {
      const uint4 ev = *reinterpret_cast<const uint4*>(er + c);
      const uint4 bv = *reinterpret_cast<const uint4*>(br + c);
      const uint32_t ew[4] = {ev.x, ev.y, ev.z, ev.w};
      const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 bf = half2_to_float2(bw[k]);
        acc = fmaf(bf16_lo(ew[k]), bf.x, acc);
        acc = fmaf(bf16_hi(ew[k]), bf.y, acc);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
    if (lane == 0) code[w] = acc;
  }
}

constexpr int kCodeRows = 128;  // timesteps whose codes are staged in shared memory at once

// mod [L, bt, n] = proj [L, n, r] . code [bt, r]^T + bias [L, n]; r = 8 * RC.
template <int RC>
__global__ void __launch_bounds__(256) adaln_mod_kernel(const uint16_t* __restrict__ proj,
                                                        const uint16_t* __restrict__ bias,
                                                        const float* __restrict__ code, int64_t bt, int64_t L,
                                                        int64_t n, float* __restrict__ mod) {
  constexpr int R = 8 * RC;
  __shared__ float code_s[kCodeRows * R];
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const bool live = idx < L * n;
  const int64_t l = live ? idx / n : 0, i = live ? idx % n : 0;
  // The projection row and bias do not depend on the code kernel: load them first.
  float p[R];
  float c0 = 0.0f;
  if (live) {
    const uint4* pr = reinterpret_cast<const uint4*>(proj + idx * R);
#pragma unroll
    for (int q = 0; q < RC; ++q) {
      const uint4 v = pr[q];
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = half2_to_float2(w[k]);
        p[8 * q + 2 * k] = f.x;
        p[8 * q + 2 * k + 1] = f.y;
      }
    }
    if (bias != nullptr) c0 = __half2float(__ushort_as_half(bias[idx]));
  } else {
#pragma unroll
    for (int j = 0; j < R; ++j) p[j] = 0.0f;
  }
  // The codes are written by the preceding grid.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  for (int64_t b0 = 0; b0 < bt; b0 += kCodeRows) {
    const int rows = (int)(bt - b0 < kCodeRows ? bt - b0 : kCodeRows);
    __syncthreads();  // the previous chunk's codes are no longer read
    for (int t = threadIdx.x; t < rows * R; t += blockDim.x) code_s[t] = code[b0 * R + t];
    __syncthreads();
    if (live) {
      float* out = mod + (l * bt + b0) * n + i;
      for (int b = 0; b < rows; ++b) {
        const float* z = code_s + b * R;
        float acc = c0;
#pragma unroll
        for (int j = 0; j < R; ++j) acc = fmaf(p[j], z[j], acc);
        out[(int64_t)b * n] = acc;
      }
    }
  }
}

template <int RC>
cudaError_t launch_mod(const uint16_t* proj, const uint16_t* bias, const float* code, int64_t bt, int64_t L,
                       int64_t n, float* mod, cudaStream_t s) {
  const int64_t threads = L * n;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((threads + 255) / 256));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, adaln_mod_kernel<RC>, proj, bias, code, bt, L, n, mod);
}

}  // namespace

cudaError_t launch_adaln_modulation(const uint16_t* e, int64_t bt, int64_t d, const uint16_t* basis, int64_t r,
                                    const uint16_t* proj, const uint16_t* bias, int64_t L, int64_t n, float* code,
                                    float* mod, cudaStream_t s) {
  const int64_t warps_needed = bt * r;
  const int64_t cap = (int64_t)sm_count() * 8;
  const int64_t blocks = (warps_needed + 7) / 8;
  const int grid = (int)(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
  adaln_code_kernel<<<grid, 256, 0, s>>>(e, bt, d, basis, (int)r, code);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  if (L * n == 0) return cudaSuccess;  // only the codes were asked for
  switch (r) {
    case 8: return launch_mod<1>(proj, bias, code, bt, L, n, mod, s);
    case 16: return launch_mod<2>(proj, bias, code, bt, L, n, mod, s);
    case 24: return launch_mod<3>(proj, bias, code, bt, L, n, mod, s);
    default: return launch_mod<4>(proj, bias, code, bt, L, n, mod, s);
  }
}

}  // namespace fh
