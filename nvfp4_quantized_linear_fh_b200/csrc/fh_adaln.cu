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
//   adaln_code_kernel  one CTA per (b, four basis rows): independent 16-byte
//                      loads across the CTA, then a block reduction.  It lets
//                      the dependent grid start at once.
//   adaln_mod_kernel   one resident wave of CTAs walking groups of projection
//                      rows (two per thread); each thread's FP16 rows and
//                      biases for the first group are read before
//                      griddepcontrol.wait, so that this HBM read overlaps the
//                      code kernel, and the next group's are in flight while
//                      the current one is computed.  The codes are staged in
//                      shared memory once per CTA (128 timesteps at a time),
//                      interleaved by timestep pairs so that packed FP32 FMAs
//                      evaluate two timesteps per instruction, and each
//                      timestep's row of modulations is written with coalesced
//                      FP32 stores.
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

// code [bt, r] = e [bt, d] . basis^T, basis [r, d]; d % 8 == 0.  Block (b, g)
// computes code[b, 4g .. 4g+3]: every thread loads its 16-byte chunks of the
// embedding row and of the four basis rows at once (no dependent loads), then
// the block reduces the four partial sums.
constexpr int kCodeThreads = 256;
__global__ void __launch_bounds__(kCodeThreads) adaln_code_kernel(const uint16_t* __restrict__ e, int64_t d,
                                                                  const uint16_t* __restrict__ basis, int r,
                                                                  float* __restrict__ code) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ float part[kCodeThreads / 32][4];
  const int64_t b = blockIdx.x;
  const int j0 = 4 * blockIdx.y;
  const uint16_t* er = e + b * d;
  float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  for (int64_t c = 8 * (int64_t)threadIdx.x; c < d; c += 8 * kCodeThreads) {
    const uint4 ev = *reinterpret_cast<const uint4*>(er + c);
    uint4 bv[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) bv[q] = *reinterpret_cast<const uint4*>(basis + (int64_t)(j0 + q) * d + c);
    const uint32_t ew[4] = {ev.x, ev.y, ev.z, ev.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t bw[4] = {bv[q].x, bv[q].y, bv[q].z, bv[q].w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 bf = half2_to_float2(bw[k]);
        acc[q] = fmaf(bf16_lo(ew[k]), bf.x, acc[q]);
        acc[q] = fmaf(bf16_hi(ew[k]), bf.y, acc[q]);
      }
    }
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc[q] += __shfl_xor_sync(0xFFFFFFFFu, acc[q], o);
  }
  if (lane == 0) {
#pragma unroll
    for (int q = 0; q < 4; ++q) part[warp][q] = acc[q];
  }
  __syncthreads();
  if (threadIdx.x < 4) {
    float t = 0.0f;
#pragma unroll
    for (int w = 0; w < kCodeThreads / 32; ++w) t += part[w][threadIdx.x];
    code[b * r + j0 + threadIdx.x] = t;
  }
}

constexpr int kCodeRows = 128;  // timesteps whose codes are staged in shared memory at once
constexpr int kModThreads = 256;
constexpr int kModRows = 2;     // projection rows per thread per group

// mod [L, bt, n] = proj [L, n, r] . code [bt, r]^T + bias [L, n]; r = 8 * RC.
// Row groups of kModThreads * kModRows rows are walked grid-stride; a thread
// holds the raw FP16 rows of its current group and has the next group's in
// flight.  The first group is loaded before griddepcontrol.wait.
template <int RC>
__global__ void __launch_bounds__(kModThreads) adaln_mod_kernel(const uint16_t* __restrict__ proj,
                                                                const uint16_t* __restrict__ bias,
                                                                const float* __restrict__ code, int64_t bt,
                                                                int64_t rows_total, int64_t n,
                                                                float* __restrict__ mod) {
  constexpr int R = 8 * RC;
  constexpr int64_t kGroup = (int64_t)kModThreads * kModRows;
  // Codes of timestep pairs interleaved, [b / 2][j][b % 2], so that one 16-byte
  // load gives (z[b][j], z[b+1][j], z[b][j+1], z[b+1][j+1]) for packed FMAs.
  __shared__ float4 code_s[kCodeRows / 2 * R / 2];
  struct Raw {
    uint4 w[kModRows][RC];
    uint16_t c[kModRows];
  };
  auto fetch = [&](int64_t g, Raw& raw) {
#pragma unroll
    for (int k = 0; k < kModRows; ++k) {
      const int64_t idx = g * kGroup + (int64_t)k * kModThreads + threadIdx.x;
      const bool live = idx < rows_total;
      const uint4* pr = reinterpret_cast<const uint4*>(proj + (live ? idx : 0) * R);
#pragma unroll
      for (int q = 0; q < RC; ++q) raw.w[k][q] = live ? pr[q] : make_uint4(0, 0, 0, 0);
      raw.c[k] = (live && bias != nullptr) ? bias[idx] : (uint16_t)0;
    }
  };
  const int64_t groups = (rows_total + kGroup - 1) / kGroup;
  Raw cur, nxt;
  // The projections do not depend on the code kernel: start reading them now.
  if ((int64_t)blockIdx.x < groups) fetch(blockIdx.x, cur);
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the codes are written by the preceding grid
  for (int64_t b0 = 0; b0 < bt; b0 += kCodeRows) {
    const int nb = (int)(bt - b0 < kCodeRows ? bt - b0 : kCodeRows);
    const int npairs = (nb + 1) / 2;
    __syncthreads();  // the previous chunk's codes are no longer read
    float* cs = reinterpret_cast<float*>(code_s);
    for (int t = threadIdx.x; t < npairs * 2 * R; t += kModThreads) {
      const int bb = 2 * (t / (2 * R)) + (t & 1), j = (t % (2 * R)) >> 1;
      cs[t] = bb < nb ? code[(b0 + bb) * R + j] : 0.0f;  // an odd count pads with zeros
    }
    __syncthreads();
    if (b0 > 0 && (int64_t)blockIdx.x < groups) fetch(blockIdx.x, cur);  // later chunks re-read (from L2)
    for (int64_t g = blockIdx.x; g < groups; g += gridDim.x) {
      if (g + gridDim.x < groups) fetch(g + gridDim.x, nxt);
      float2 pp[kModRows][R];  // (p_j, p_j): the weight against both timesteps of a pair
      float2 c2[kModRows];
      float* out[kModRows];
      bool live[kModRows];
#pragma unroll
      for (int k = 0; k < kModRows; ++k) {
        const int64_t idx = g * kGroup + (int64_t)k * kModThreads + threadIdx.x;
        live[k] = idx < rows_total;
#pragma unroll
        for (int q = 0; q < RC; ++q) {
          const uint32_t w[4] = {cur.w[k][q].x, cur.w[k][q].y, cur.w[k][q].z, cur.w[k][q].w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const float2 f = half2_to_float2(w[h]);
            pp[k][8 * q + 2 * h] = make_float2(f.x, f.x);
            pp[k][8 * q + 2 * h + 1] = make_float2(f.y, f.y);
          }
        }
        const float c0 = __half2float(__ushort_as_half(cur.c[k]));
        c2[k] = make_float2(c0, c0);
        const uint32_t row = live[k] ? (uint32_t)idx : 0u;  // rows_total < 2^31
        const uint32_t l = row / (uint32_t)n, i = row - l * (uint32_t)n;
        out[k] = mod + ((int64_t)l * bt + b0) * n + i;
      }
      for (int bp = 0; bp < npairs; ++bp) {
        float2 acc[kModRows];
#pragma unroll
        for (int k = 0; k < kModRows; ++k) acc[k] = c2[k];
#pragma unroll
        for (int jq = 0; jq < R / 2; ++jq) {
          const float4 zz = code_s[bp * (R / 2) + jq];
#pragma unroll
          for (int k = 0; k < kModRows; ++k) {
            acc[k] = __ffma2_rn(pp[k][2 * jq], make_float2(zz.x, zz.y), acc[k]);
            acc[k] = __ffma2_rn(pp[k][2 * jq + 1], make_float2(zz.z, zz.w), acc[k]);
          }
        }
        const int b = 2 * bp;
#pragma unroll
        for (int k = 0; k < kModRows; ++k) {
          if (!live[k]) continue;
          out[k][(int64_t)b * n] = acc[k].x;
          if (b + 1 < nb) out[k][(int64_t)(b + 1) * n] = acc[k].y;
        }
      }
      cur = nxt;
    }
  }
}

template <int RC>
cudaError_t launch_mod(const uint16_t* proj, const uint16_t* bias, const float* code, int64_t bt, int64_t L,
                       int64_t n, float* mod, cudaStream_t s) {
  const int64_t rows_total = L * n;
  const int64_t groups = (rows_total + (int64_t)kModThreads * kModRows - 1) / ((int64_t)kModThreads * kModRows);
  static DeviceTable resident;  // resident CTAs per SM for this instantiation (one wave)
  int dev = 0;
  cudaGetDevice(&dev);
  const int per_sm = per_device(resident, dev, [](int) {
    int n = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, adaln_mod_kernel<RC>, kModThreads, 0);
    return e != cudaSuccess ? -(int)e : (n < 1 ? 1 : n);
  });
  if (per_sm <= 0) return (cudaError_t)(-per_sm);
  const int64_t cap = (int64_t)sm_count() * per_sm;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(groups < cap ? groups : cap));
  cfg.blockDim = dim3(kModThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, adaln_mod_kernel<RC>, proj, bias, code, bt, rows_total, n, mod);
}

}  // namespace

cudaError_t launch_adaln_modulation(const uint16_t* e, int64_t bt, int64_t d, const uint16_t* basis, int64_t r,
                                    const uint16_t* proj, const uint16_t* bias, int64_t L, int64_t n, float* code,
                                    float* mod, cudaStream_t s) {
  adaln_code_kernel<<<dim3((unsigned)bt, (unsigned)(r / 4)), kCodeThreads, 0, s>>>(e, d, basis, (int)r, code);
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
