"""Python binding of libfh, the NVFP4 quantized linear layer for B200 (sm_100a).

Argument marshalling only: every function below has the name of the C entry
point it calls (include/fh.h), checks that the torch tensors it is given have
the dtype, device and contiguity the C ABI expects, passes their device
pointers and the current CUDA stream, and raises FHError on a non-zero status.
All arithmetic runs in the CUDA kernels of libfh.so.  There is no fallback:
importing this package fails if libfh.so has not been built
(``python nvfp4_quantized_linear_fh_b200/build.py``).

The layer is the NVFP4 linear layer of FastH3's diffusion transformer (FastH3
thread digest, farwalk.ai, tweets 5/8 and 6/8; FastH3 Trim, comfyui-wiki news,
"What the ComfyUI repack contains").
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfh.so")

FH_OK = 0
FH_ERR_INVALID_ARG = 1
FH_ERR_UNSUPPORTED_SHAPE = 2
FH_ERR_CUDA = 3
FH_ERR_TIMEOUT = 4
FH_ERR_NO_DEVICE = 5

FH_SCALES_ROWMAJOR = 0
FH_SCALES_MMA_TILED = 1


class FHError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"libfh status {status}: {message}")
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python nvfp4_quantized_linear_fh_b200/build.py` "
                      "(the NVFP4 layer has no CPU fallback)")

_lib = ctypes.CDLL(LIB_PATH)
_c = ctypes
_P = _c.c_void_p
_I64 = _c.c_int64
_SIG = {
    "fh_version": (_c.c_int, []),
    "fh_last_error": (_c.c_char_p, []),
    "fh_scale_from_amax": (_c.c_float, [_c.c_float]),
    "fh_scales_bytes": (_c.c_size_t, [_I64, _I64, _c.c_int]),
    "fh_amax": (_c.c_int, [_P, _I64, _I64, _I64, _P, _P]),
    "fh_quantize_act": (_c.c_int, [_P, _I64, _I64, _I64, _c.c_float, _P, _P, _P, _c.c_int, _P]),
    "fh_gelu_quantize_act": (_c.c_int, [_P, _I64, _I64, _I64, _c.c_float, _P, _P, _P, _P]),
    "fh_nvfp4_linear": (_c.c_int, [_P, _P, _c.c_float, _P, _P, _c.c_float, _P, _P, _I64, _I64, _I64, _P]),
    "fh_nvfp4_linear_gelu_quant": (_c.c_int, [_P, _P, _c.c_float, _P, _P, _c.c_float, _P, _c.c_float, _P, _P, _P,
                                              _I64, _I64, _I64, _P]),
    "fh_scales_to_rowmajor": (_c.c_int, [_P, _P, _I64, _I64, _P]),
    "fh_nvfp4_linear_fused_quant": (_c.c_int, [_P, _I64, _I64, _I64, _c.c_float, _P, _P, _c.c_float, _P, _P, _I64,
                                               _P, _P, _P, _P, _P]),
    "fh_nvfp4_linear_fused_quant_sync_bytes": (_c.c_size_t, [_I64]),
    "fh_nvfp4_linear_host": (_c.c_int, [_P, _I64, _I64, _c.c_float, _P, _P, _c.c_float, _P, _I64, _P, _P, _I64, _P,
                                        _c.c_size_t, _P]),
    "fh_nvfp4_linear_host_workspace_bytes": (_c.c_size_t, [_I64, _I64, _I64]),
    "fh_nvfp4_linear_host_noalloc": (_c.c_int, [_P, _I64, _I64, _c.c_float, _P, _P, _c.c_float, _P, _I64, _P, _P,
                                                _P]),
    "fh_gelu_bf16": (_c.c_int, [_P, _P, _I64, _P]),
    "fh_quantize_int8_rows": (_c.c_int, [_P, _I64, _I64, _I64, _P, _P, _P]),
    "fh_int8_attention_scores": (_c.c_int, [_P, _P, _P, _P, _c.c_float, _P, _I64, _I64, _I64, _I64, _P]),
    "fh_adaln_modulation": (_c.c_int, [_P, _I64, _I64, _P, _I64, _P, _P, _I64, _I64, _P, _P, _P]),
    "fh_device_status": (_c.c_int, [_P]),
    "fh_selftest_mma_rate": (_c.c_int, [_c.c_int32, _c.c_int32, _c.POINTER(_c.c_int32), _P]),
    "fh_selftest_bounded_wait": (_c.c_int, [_c.c_uint32, _P]),
}
for _name, (_res, _args) in _SIG.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


def lib():
    """The loaded ctypes library (for tests that call the C ABI directly)."""
    return _lib


def _check(status: int):
    if status != FH_OK:
        raise FHError(status, _lib.fh_last_error().decode())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return _P(stream.cuda_stream)


def _ptr(t):
    return None if t is None else _P(t.data_ptr())


def _need(t, dtypes, what, ndim=None):
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        raise TypeError(f"{what} must be a CUDA tensor")
    if t.dtype not in dtypes:
        raise TypeError(f"{what} must have dtype in {dtypes}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{what} must have {ndim} dimensions")


_BF16 = (torch.bfloat16, torch.int16, torch.uint16)
_U8 = (torch.uint8,)


# --- host entry points --------------------------------------------------------

def fh_version() -> int:
    return _lib.fh_version()


def fh_last_error() -> str:
    return _lib.fh_last_error().decode()


def fh_scale_from_amax(amax: float) -> float:
    return _lib.fh_scale_from_amax(float(amax))


def fh_scales_bytes(rows: int, K: int, layout: int = FH_SCALES_MMA_TILED) -> int:
    return _lib.fh_scales_bytes(rows, K, layout)


# --- device entry points ------------------------------------------------------

def fh_amax(x: torch.Tensor, amax: torch.Tensor, stream=None) -> None:
    """amax[0] = max(amax[0], max |x|) for BF16 x [rows, cols] (row stride x.stride(0))."""
    _need(x, _BF16, "x", 2)
    _need(amax, (torch.float32,), "amax")
    if x.stride(1) != 1:
        raise ValueError("x must have unit column stride")
    _check(_lib.fh_amax(_ptr(x), x.shape[0], x.shape[1], x.stride(0), _ptr(amax), _stream(stream)))


def fh_quantize_act(x: torch.Tensor, global_scale: float, codes: torch.Tensor, scales: torch.Tensor,
                    clip_count: torch.Tensor | None = None, scale_layout: int = FH_SCALES_MMA_TILED,
                    stream=None) -> None:
    """NVFP4-quantize BF16 x [M, K] into codes [M, K/2] and scales (see include/fh.h)."""
    _need(x, _BF16, "x", 2)
    _need(codes, _U8, "codes")
    _need(scales, _U8, "scales")
    if x.stride(1) != 1:
        raise ValueError("x must have unit column stride")
    M, K = x.shape
    if codes.numel() < M * (K // 2) or not codes.is_contiguous():
        raise ValueError("codes must be contiguous with M*K/2 bytes")
    need = fh_scales_bytes(M, K, scale_layout)
    if scales.numel() < need or not scales.is_contiguous():
        raise ValueError(f"scales must be contiguous with {need} bytes")
    if clip_count is not None:
        _need(clip_count, (torch.int64, torch.uint64), "clip_count")
    _check(_lib.fh_quantize_act(_ptr(x), M, K, x.stride(0), float(global_scale), _ptr(codes), _ptr(scales),
                                _ptr(clip_count), scale_layout, _stream(stream)))


def fh_gelu_quantize_act(x: torch.Tensor, global_scale: float, codes: torch.Tensor, scales: torch.Tensor,
                         clip_count: torch.Tensor | None = None, stream=None) -> None:
    """NVFP4 codes and tensor-core-layout scales of GELU(x) for BF16 x [M, K] (row stride x.stride(0))."""
    _need(x, _BF16, "x", 2)
    if x.stride(1) != 1:
        raise ValueError("x must be row-major (unit column stride)")
    _need(codes, _U8, "codes", 2)
    _need(scales, _U8, "scales")
    M, K = x.shape
    if tuple(codes.shape) != (M, K // 2) or not codes.is_contiguous():
        raise ValueError("codes must be a contiguous [M, K/2] uint8 tensor")
    if scales.numel() < fh_scales_bytes(M, K):
        raise ValueError("scales too small for the tensor-core scale layout")
    if clip_count is not None and (clip_count.dtype != torch.int64 or clip_count.device.type != "cuda"):
        raise TypeError("clip_count must be a CUDA int64 tensor")
    _check(_lib.fh_gelu_quantize_act(_ptr(x), M, K, x.stride(0), float(global_scale), _ptr(codes), _ptr(scales),
                                     _ptr(clip_count), _stream(stream)))


def fh_nvfp4_linear(a_codes: torch.Tensor, a_scales: torch.Tensor, a_gscale: float,
                    w_codes: torch.Tensor, w_scales: torch.Tensor, w_gscale: float,
                    bias: torch.Tensor | None, y: torch.Tensor, stream=None) -> None:
    """y[M, N] = bf16(a_g * w_g * A . W^T + bias) on the tcgen05 tensor cores."""
    for t, n in ((a_codes, "a_codes"), (w_codes, "w_codes")):
        _need(t, _U8, n, 2)
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    _need(a_scales, _U8, "a_scales")
    _need(w_scales, _U8, "w_scales")
    _need(y, _BF16, "y", 2)
    M, K = a_codes.shape[0], a_codes.shape[1] * 2
    N = w_codes.shape[0]
    if w_codes.shape[1] * 2 != K or tuple(y.shape) != (M, N) or not y.is_contiguous():
        raise ValueError("shape mismatch: a_codes [M, K/2], w_codes [N, K/2], y [M, N] contiguous")
    if a_scales.numel() < fh_scales_bytes(M, K) or w_scales.numel() < fh_scales_bytes(N, K):
        raise ValueError("scale arrays too small for the tensor-core scale layout")
    if bias is not None:
        _need(bias, _BF16, "bias")
        if bias.numel() != N or not bias.is_contiguous():
            raise ValueError("bias must be contiguous with N elements")
    _check(_lib.fh_nvfp4_linear(_ptr(a_codes), _ptr(a_scales), float(a_gscale), _ptr(w_codes), _ptr(w_scales),
                                float(w_gscale), _ptr(bias), _ptr(y), M, N, K, _stream(stream)))


def fh_nvfp4_linear_gelu_quant(a_codes: torch.Tensor, a_scales: torch.Tensor, a_gscale: float,
                               w_codes: torch.Tensor, w_scales: torch.Tensor, w_gscale: float,
                               bias: torch.Tensor | None, out_gscale: float, out_codes: torch.Tensor,
                               out_scales: torch.Tensor, out_clip: torch.Tensor | None = None, stream=None) -> None:
    """NVFP4 input of the next layer, GELU(bf16(a_g * w_g * A . W^T + bias)) quantized with out_gscale,
    written as out_codes [M, N/2] and tensor-core-layout out_scales; out_clip (int64, 1 element) += clips."""
    for t, n in ((a_codes, "a_codes"), (w_codes, "w_codes"), (out_codes, "out_codes")):
        _need(t, _U8, n, 2)
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    _need(a_scales, _U8, "a_scales")
    _need(w_scales, _U8, "w_scales")
    _need(out_scales, _U8, "out_scales")
    M, K = a_codes.shape[0], a_codes.shape[1] * 2
    N = w_codes.shape[0]
    if w_codes.shape[1] * 2 != K or tuple(out_codes.shape) != (M, N // 2):
        raise ValueError("shape mismatch: a_codes [M, K/2], w_codes [N, K/2], out_codes [M, N/2]")
    if (a_scales.numel() < fh_scales_bytes(M, K) or w_scales.numel() < fh_scales_bytes(N, K)
            or out_scales.numel() < fh_scales_bytes(M, N)):
        raise ValueError("scale arrays too small for the tensor-core scale layout")
    if bias is not None:
        _need(bias, _BF16, "bias")
        if bias.numel() != N or not bias.is_contiguous():
            raise ValueError("bias must be contiguous with N elements")
    if out_clip is not None and (out_clip.dtype != torch.int64 or out_clip.device.type != "cuda"):
        raise TypeError("out_clip must be a CUDA int64 tensor")
    _check(_lib.fh_nvfp4_linear_gelu_quant(_ptr(a_codes), _ptr(a_scales), float(a_gscale), _ptr(w_codes),
                                           _ptr(w_scales), float(w_gscale), _ptr(bias), float(out_gscale),
                                           _ptr(out_codes), _ptr(out_scales), _ptr(out_clip), M, N, K,
                                           _stream(stream)))


def fh_nvfp4_linear_fused_quant_sync_bytes(M: int) -> int:
    return _lib.fh_nvfp4_linear_fused_quant_sync_bytes(M)


def empty_fused_sync(M: int, device="cuda") -> torch.Tensor:
    """A zeroed sync buffer for fh_nvfp4_linear_fused_quant (each call leaves it zero again)."""
    return torch.zeros(max(1, fh_nvfp4_linear_fused_quant_sync_bytes(M) // 4), dtype=torch.int32, device=device)


def fh_nvfp4_linear_fused_quant(x: torch.Tensor, a_gscale: float, w_codes: torch.Tensor, w_scales: torch.Tensor,
                                w_gscale: float, bias: torch.Tensor | None, y: torch.Tensor, a_codes: torch.Tensor,
                                a_scales: torch.Tensor, clip: torch.Tensor | None, sync: torch.Tensor,
                                stream=None) -> None:
    """y [M, N] = the NVFP4 layer on BF16 x [M, K] with the quantization in the same kernel; also writes x's
    codes and tensor-core-layout scales into a_codes / a_scales (see include/fh.h).  sync: empty_fused_sync(M)."""
    _need(x, _BF16, "x", 2)
    _need(w_codes, _U8, "w_codes", 2)
    _need(w_scales, _U8, "w_scales")
    _need(y, _BF16, "y", 2)
    _need(a_codes, _U8, "a_codes", 2)
    _need(a_scales, _U8, "a_scales")
    _need(sync, (torch.int32, torch.uint32), "sync")
    if x.stride(1) != 1 or not (y.is_contiguous() and a_codes.is_contiguous() and w_codes.is_contiguous()):
        raise ValueError("x rows must be contiguous; y, a_codes, w_codes contiguous")
    M, K = x.shape
    N = w_codes.shape[0]
    if w_codes.shape[1] * 2 != K or tuple(y.shape) != (M, N) or tuple(a_codes.shape) != (M, K // 2):
        raise ValueError("shape mismatch: x [M, K], w_codes [N, K/2], y [M, N], a_codes [M, K/2]")
    if a_scales.numel() < fh_scales_bytes(M, K, FH_SCALES_MMA_TILED):
        raise ValueError("a_scales too small")
    if sync.numel() * 4 < fh_nvfp4_linear_fused_quant_sync_bytes(M):
        raise ValueError("sync too small")
    if bias is not None:
        _need(bias, _BF16, "bias")
    if clip is not None and (clip.dtype != torch.int64 or clip.device.type != "cuda"):
        raise TypeError("clip must be a CUDA int64 tensor")
    _check(_lib.fh_nvfp4_linear_fused_quant(_ptr(x), M, K, x.stride(0), float(a_gscale), _ptr(w_codes),
                                            _ptr(w_scales), float(w_gscale), _ptr(bias), _ptr(y), N, _ptr(a_codes),
                                            _ptr(a_scales), _ptr(clip), _ptr(sync), _stream(stream)))


def fh_nvfp4_linear_host_workspace_bytes(K: int, N: int, chunk_rows: int = 4096) -> int:
    return _lib.fh_nvfp4_linear_host_workspace_bytes(K, N, chunk_rows)


def fh_nvfp4_linear_host(x_host: torch.Tensor, a_gscale: float, w_codes: torch.Tensor, w_scales: torch.Tensor,
                         w_gscale: float, bias: torch.Tensor | None, y_host: torch.Tensor,
                         clip: torch.Tensor | None = None, chunk_rows: int = 4096,
                         workspace: torch.Tensor | None = None, stream=None) -> None:
    """y_host [M, N] = the NVFP4 layer on x_host [M, K]: host BF16 tensors (pin them for overlap), weights on the
    device; chunked upload, quantize, GEMM and download overlap (see include/fh.h).  Ordered on the stream:
    synchronize before reading y_host.  workspace: CUDA uint8 of fh_nvfp4_linear_host_workspace_bytes bytes, or
    None to allocate one for this call."""
    for t, n in ((x_host, "x_host"), (y_host, "y_host")):
        if not isinstance(t, torch.Tensor) or t.device.type != "cpu" or t.dtype not in _BF16 or t.dim() != 2:
            raise TypeError(f"{n} must be a 2-D BF16 CPU tensor")
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    _need(w_codes, _U8, "w_codes", 2)
    _need(w_scales, _U8, "w_scales")
    M, K = x_host.shape
    N = w_codes.shape[0]
    if w_codes.shape[1] * 2 != K or tuple(y_host.shape) != (M, N):
        raise ValueError("shape mismatch: x_host [M, K], w_codes [N, K/2], y_host [M, N]")
    if bias is not None:
        _need(bias, _BF16, "bias")
    if clip is not None and (clip.dtype != torch.int64 or clip.device.type != "cuda"):
        raise TypeError("clip must be a CUDA int64 tensor")
    need = fh_nvfp4_linear_host_workspace_bytes(K, N, chunk_rows)
    own = workspace is None
    if own:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=w_codes.device)
    _need(workspace, _U8, "workspace")
    torch_stream = torch.cuda.current_stream(w_codes.device) if stream is None else stream
    _check(_lib.fh_nvfp4_linear_host(_P(x_host.data_ptr()), M, K, float(a_gscale), _ptr(w_codes), _ptr(w_scales),
                                     float(w_gscale), _ptr(bias), N, _P(y_host.data_ptr()), _ptr(clip), chunk_rows,
                                     _ptr(workspace), workspace.numel(), _stream(torch_stream)))
    if own:
        # The call's work on `stream` still uses the workspace after this returns:
        # the caching allocator must not hand the block to other streams before
        # that work has finished.
        workspace.record_stream(torch_stream)


def fh_nvfp4_linear_host_noalloc(x_host: torch.Tensor, a_gscale: float, w_codes: torch.Tensor,
                                 w_scales: torch.Tensor, w_gscale: float, bias: torch.Tensor | None,
                                 y_host: torch.Tensor, clip: torch.Tensor | None = None, stream=None) -> None:
    """fh_nvfp4_linear_host without a workspace: the chunks are staged in the library's static device scratch
    array (see include/fh.h), so nothing is allocated on the device.  Calls sharing a device must not overlap on
    the GPU.  Ordered on the stream: synchronize before reading y_host."""
    for t, n in ((x_host, "x_host"), (y_host, "y_host")):
        if not isinstance(t, torch.Tensor) or t.device.type != "cpu" or t.dtype not in _BF16 or t.dim() != 2:
            raise TypeError(f"{n} must be a 2-D BF16 CPU tensor")
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    _need(w_codes, _U8, "w_codes", 2)
    _need(w_scales, _U8, "w_scales")
    M, K = x_host.shape
    N = w_codes.shape[0]
    if w_codes.shape[1] * 2 != K or tuple(y_host.shape) != (M, N):
        raise ValueError("shape mismatch: x_host [M, K], w_codes [N, K/2], y_host [M, N]")
    if bias is not None:
        _need(bias, _BF16, "bias")
    if clip is not None and (clip.dtype != torch.int64 or clip.device.type != "cuda"):
        raise TypeError("clip must be a CUDA int64 tensor")
    _check(_lib.fh_nvfp4_linear_host_noalloc(_P(x_host.data_ptr()), M, K, float(a_gscale), _ptr(w_codes),
                                             _ptr(w_scales), float(w_gscale), _ptr(bias), N, _P(y_host.data_ptr()),
                                             _ptr(clip), _stream(stream)))


def fh_scales_to_rowmajor(tiled: torch.Tensor, rowmajor: torch.Tensor, rows: int, K: int, stream=None) -> None:
    _need(tiled, _U8, "tiled")
    _need(rowmajor, _U8, "rowmajor")
    if rowmajor.numel() < rows * (K // 16) or tiled.numel() < fh_scales_bytes(rows, K):
        raise ValueError("buffer too small")
    _check(_lib.fh_scales_to_rowmajor(_ptr(tiled), _ptr(rowmajor), rows, K, _stream(stream)))


def fh_gelu_bf16(x: torch.Tensor, y: torch.Tensor, stream=None) -> None:
    _need(x, _BF16, "x")
    _need(y, _BF16, "y")
    if x.numel() != y.numel() or not x.is_contiguous() or not y.is_contiguous():
        raise ValueError("x and y must be contiguous with the same number of elements")
    _check(_lib.fh_gelu_bf16(_ptr(x), _ptr(y), x.numel(), _stream(stream)))


def fh_quantize_int8_rows(x: torch.Tensor, q: torch.Tensor, scales: torch.Tensor, stream=None) -> None:
    """Per-row symmetric INT8: BF16 x [rows, d] (row stride x.stride(0)) -> q int8 [rows, d], scales FP32 [rows]."""
    _need(x, _BF16, "x", 2)
    _need(q, (torch.int8,), "q", 2)
    _need(scales, (torch.float32,), "scales", 1)
    rows, d = x.shape
    if x.stride(1) != 1 or not q.is_contiguous() or not scales.is_contiguous():
        raise ValueError("x needs unit column stride; q and scales must be contiguous")
    if tuple(q.shape) != (rows, d) or scales.numel() != rows:
        raise ValueError("shape mismatch: q [rows, d], scales [rows]")
    _check(_lib.fh_quantize_int8_rows(_ptr(x), rows, d, x.stride(0), _ptr(q), _ptr(scales), _stream(stream)))


def fh_int8_attention_scores(q: torch.Tensor, q_scales: torch.Tensor, k: torch.Tensor, k_scales: torch.Tensor,
                             sm_scale: float, s: torch.Tensor, stream=None) -> None:
    """S [heads, tq, tk] FP32 = (acc * (s_q * sm_scale)) * s_k for INT8 q [heads, tq, d], k [heads, tk, d]."""
    _need(q, (torch.int8,), "q", 3)
    _need(k, (torch.int8,), "k", 3)
    _need(q_scales, (torch.float32,), "q_scales")
    _need(k_scales, (torch.float32,), "k_scales")
    _need(s, (torch.float32,), "s", 3)
    for t, n in ((q, "q"), (k, "k"), (q_scales, "q_scales"), (k_scales, "k_scales"), (s, "s")):
        if not t.is_contiguous():
            raise ValueError(f"{n} must be contiguous")
    heads, tq, d = q.shape
    tk = k.shape[1]
    if (k.shape[0] != heads or k.shape[2] != d or tuple(s.shape) != (heads, tq, tk)
            or q_scales.numel() != heads * tq or k_scales.numel() != heads * tk):
        raise ValueError("shape mismatch: q [H, tq, d], k [H, tk, d], scales [H, t], s [H, tq, tk]")
    _check(_lib.fh_int8_attention_scores(_ptr(q), _ptr(q_scales), _ptr(k), _ptr(k_scales), float(sm_scale),
                                         _ptr(s), heads, tq, tk, d, _stream(stream)))


def fh_adaln_modulation(temb: torch.Tensor, basis: torch.Tensor, proj: torch.Tensor, bias: torch.Tensor | None,
                        code: torch.Tensor, mod: torch.Tensor, stream=None) -> None:
    """code [bt, r] = temb [bt, d] . basis^T (basis [r, d] FP16); mod [blocks, bt, n] = proj [blocks, n, r] . code^T
    + bias [blocks, n], all FP32 results."""
    _need(temb, _BF16, "temb", 2)
    _need(basis, (torch.float16,), "basis", 2)
    _need(proj, (torch.float16,), "proj", 3)
    _need(code, (torch.float32,), "code", 2)
    _need(mod, (torch.float32,), "mod", 3)
    if bias is not None:
        _need(bias, (torch.float16,), "bias", 2)
    for t, nm in ((temb, "temb"), (basis, "basis"), (proj, "proj"), (code, "code"), (mod, "mod"), (bias, "bias")):
        if t is not None and not t.is_contiguous():
            raise ValueError(f"{nm} must be contiguous")
    bt, d = temb.shape
    r = basis.shape[0]
    blocks, n = proj.shape[0], proj.shape[1]
    if (basis.shape[1] != d or proj.shape[2] != r or tuple(code.shape) != (bt, r)
            or tuple(mod.shape) != (blocks, bt, n) or (bias is not None and tuple(bias.shape) != (blocks, n))):
        raise ValueError("shape mismatch: temb [bt, d], basis [r, d], proj [blocks, n, r], bias [blocks, n], "
                         "code [bt, r], mod [blocks, bt, n]")
    _check(_lib.fh_adaln_modulation(_ptr(temb), bt, d, _ptr(basis), r, _ptr(proj), _ptr(bias), blocks, n,
                                    _ptr(code), _ptr(mod), _stream(stream)))


def fh_selftest_bounded_wait(limit_us: int, stream=None) -> None:
    """Enqueue the bounded-wait self-test (see include/fh.h); fh_device_status then reports the timeout."""
    _check(_lib.fh_selftest_bounded_wait(int(limit_us), _stream(stream)))


def fh_selftest_mma_rate(iters: int, with_scale_copies: bool = False, stream=None) -> int:
    """Enqueue the FP4 tensor-rate probe (see include/fh.h); returns the number of CTA pairs.
    Each pair performs iters * 2 * 256 * 256 * 256 FLOP."""
    pairs = _c.c_int32(0)
    _check(_lib.fh_selftest_mma_rate(int(iters), 1 if with_scale_copies else 0, _c.byref(pairs), _stream(stream)))
    return pairs.value


def fh_device_status(stream=None) -> None:
    """Synchronize and raise FHError(FH_ERR_TIMEOUT) if a kernel gave up on a bounded wait."""
    _check(_lib.fh_device_status(_stream(stream)))


# --- allocation helpers (marshalling only) ----------------------------------------

def empty_quantized(rows: int, K: int, device="cuda", layout: int = FH_SCALES_MMA_TILED):
    """Uninitialised (codes [rows, K/2], scales) buffers for fh_quantize_act."""
    codes = torch.empty((rows, K // 2), dtype=torch.uint8, device=device)
    scales = torch.empty(max(fh_scales_bytes(rows, K, layout), 1), dtype=torch.uint8, device=device)
    return codes, scales
