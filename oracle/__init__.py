"""CPU oracle of the NVFP4 quantized linear layer (binding to fh_oracle.c), and
numpy definitions of the INT8 query/key scores and of the AdaLN basis projection.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference legs may import this package.  It shares
no code with the CUDA library and imports nothing from it.

Every function states the definition it computes; fh_oracle.c carries the
citations (FastH3 thread digest, farwalk.ai, tweets 5/8 and 6/8; FastH3 Trim,
comfyui-wiki news, "What the ComfyUI repack contains").
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fh_oracle.c")
_LIB = os.path.join(_HERE, "libfh_oracle.so")

#: Largest magnitude of the scaled format: 6 (E2M1) * 448 (E4M3).
FORMAT_MAX = 2688.0


def build(force: bool = False) -> str:
    """Compile fh_oracle.c with gcc (plain -O2, OpenMP, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-shared", "-fPIC", "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        c = ctypes
        L.oracle_bf16_value.restype = c.c_double
        L.oracle_bf16_value.argtypes = [c.c_uint16]
        L.oracle_e2m1_value.restype = c.c_double
        L.oracle_e2m1_value.argtypes = [c.c_int]
        L.oracle_e4m3_value.restype = c.c_double
        L.oracle_e4m3_value.argtypes = [c.c_int]
        L.oracle_e4m3_rne_sat.restype = c.c_int
        L.oracle_e4m3_rne_sat.argtypes = [c.c_double]
        L.oracle_e2m1_rne_sat.restype = c.c_int
        L.oracle_e2m1_rne_sat.argtypes = [c.c_double]
        L.oracle_scale_from_amax.restype = c.c_float
        L.oracle_scale_from_amax.argtypes = [c.c_float]
        L.oracle_amax.restype = c.c_float
        L.oracle_amax.argtypes = [c.c_void_p, c.c_int64, c.c_int64, c.c_int64]
        L.oracle_quantize.restype = None
        L.oracle_quantize.argtypes = [c.c_void_p, c.c_int64, c.c_int64, c.c_int64, c.c_float,
                                      c.c_void_p, c.c_void_p, c.c_void_p]
        L.oracle_clip_count.restype = c.c_uint64
        L.oracle_clip_count.argtypes = [c.c_void_p, c.c_int64, c.c_int64, c.c_int64, c.c_float]
        L.oracle_linear.restype = None
        L.oracle_linear.argtypes = [c.c_void_p, c.c_void_p, c.c_float, c.c_void_p, c.c_void_p, c.c_float,
                                    c.c_void_p, c.c_int64, c.c_int64, c.c_void_p, c.c_int64,
                                    c.c_void_p, c.c_void_p, c.c_void_p, c.c_void_p]
        L.oracle_gelu.restype = None
        L.oracle_gelu.argtypes = [c.c_void_p, c.c_int64, c.c_void_p]
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


# --- element formats --------------------------------------------------------

def bf16_value(bits: int) -> float:
    return lib().oracle_bf16_value(bits)


def e2m1_value(code: int) -> float:
    """Value of a 4-bit E2M1 code (bit 3 sign; magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6)."""
    return lib().oracle_e2m1_value(code)


def e4m3_value(byte: int) -> float:
    """Value of an E4M3 (FN) byte; NaN for 0x7F / 0xFF."""
    return lib().oracle_e4m3_value(byte)


def e4m3_rne_sat(q: float) -> int:
    """E4M3 code of q >= 0: nearest, ties to even, q >= 448 gives 448."""
    return lib().oracle_e4m3_rne_sat(q)


def e2m1_rne_sat(r: float) -> int:
    """E2M1 magnitude code of r >= 0: nearest, ties to even, saturating at 6."""
    return lib().oracle_e2m1_rne_sat(r)


# --- calibration -------------------------------------------------------------

def scale_from_amax(amax: float) -> float:
    """Smallest FP32 s_g with 2688 * s_g >= amax (1.0 for amax == 0)."""
    return lib().oracle_scale_from_amax(float(amax))


def amax(x_bits: np.ndarray) -> float:
    """max |x| over a BF16 matrix given as uint16 bits [rows, cols]."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    if x.ndim == 1:
        x = x.reshape(1, -1)
    return lib().oracle_amax(_ptr(x), x.shape[0], x.shape[1], x.shape[1])


# --- quantization ----------------------------------------------------------

def quantize(x_bits: np.ndarray, sg: float):
    """Quantize BF16 x [M, K] (K % 16 == 0) with global scale sg.

    Returns (codes [M, K/2] uint8 with element 2j in the low nibble,
             scales [M, K/16] uint8 E4M3, row-major,
             clip count: elements with |x| > 2688 * sg)."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    M, K = x.shape
    assert K % 16 == 0
    codes = np.empty((M, K // 2), dtype=np.uint8)
    scales = np.empty((M, K // 16), dtype=np.uint8)
    clip = np.zeros(1, dtype=np.uint64)
    lib().oracle_quantize(_ptr(x), M, K, K, float(sg), _ptr(codes), _ptr(scales), _ptr(clip))
    return codes, scales, int(clip[0])


def clip_count(x_bits: np.ndarray, sg: float) -> int:
    """Number of elements of BF16 x (uint16 bits, any 2-D shape) with
    |x| > 2688 * sg: the clip count of quantize(x, sg) without the codes."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    if x.ndim == 1:
        x = x.reshape(1, -1)
    return int(lib().oracle_clip_count(_ptr(x), x.shape[0], x.shape[1], x.shape[1], float(sg)))


def tiled_scale_offsets(rows: int, K: int) -> np.ndarray:
    """Byte offset, in the tensor-core (MMA-tiled) scale layout, of scale (r, s)
    for r < rows, s < K/16.

    The layout is the one the block-scaled tensor-core MMA reads: rows are
    padded to a multiple of 128 and scale columns to a multiple of 4; the
    matrix is cut into atoms of 128 rows x 4 scales (512 bytes), atoms ordered
    with the K-atom index fastest; inside an atom, row r = r0 + 32 r1
    (r0 < 32, r1 < 4) and scale column s = 4 k1 + k0 sit at byte
    r0 * 16 + r1 * 4 + k0."""
    ns = K // 16
    ka = -(-ns // 4)
    r = np.arange(rows)[:, None]
    s = np.arange(ns)[None, :]
    atom = (r // 128) * ka + s // 4
    rr = r % 128
    return atom * 512 + (rr % 32) * 16 + (rr // 32) * 4 + s % 4


def tiled_scales_bytes(rows: int, K: int) -> int:
    return (-(-rows // 128)) * 128 * (-(-(K // 16) // 4)) * 4


# --- linear layer ------------------------------------------------------------

def linear(a_codes, a_scales, a_g, w_codes, w_scales, w_g, bias_bits, rows=None):
    """y = a_g * w_g * (A_deq . W_deq^T) + bias in binary64, on the requested rows.

    Returns (y [len(rows), N], mag [len(rows), N]) where mag is
    |a_g * w_g| * sum_k |A_deq[m,k] * W_deq[n,k]| (the error-bound magnitude)."""
    a_codes = np.ascontiguousarray(a_codes, dtype=np.uint8)
    a_scales = np.ascontiguousarray(a_scales, dtype=np.uint8)
    w_codes = np.ascontiguousarray(w_codes, dtype=np.uint8)
    w_scales = np.ascontiguousarray(w_scales, dtype=np.uint8)
    M, K = a_codes.shape[0], a_codes.shape[1] * 2
    N = w_codes.shape[0]
    rows = np.arange(M, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    b = None if bias_bits is None else np.ascontiguousarray(bias_bits, dtype=np.uint16)
    y = np.empty((rows.size, N), dtype=np.float64)
    mag = np.empty((rows.size, N), dtype=np.float64)
    w_deq = np.empty((N, K), dtype=np.float64)
    a_deq = np.empty((rows.size, K), dtype=np.float64)
    lib().oracle_linear(_ptr(a_codes), _ptr(a_scales), float(a_g), _ptr(w_codes), _ptr(w_scales), float(w_g),
                        None if b is None else _ptr(b), N, K, _ptr(rows), rows.size,
                        _ptr(w_deq), _ptr(a_deq), _ptr(y), _ptr(mag))
    return y, mag


def linear_tolerance(y_ref: np.ndarray, mag: np.ndarray) -> np.ndarray:
    """Allowed |y - y_ref| of a BF16 output: 2^-8 |y_ref| + 1e-5 * mag."""
    return np.abs(y_ref) * 2.0 ** -8 + 1e-5 * mag


def gelu(x_bits: np.ndarray) -> np.ndarray:
    """Exact-erf GELU of BF16 inputs, in binary64."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16).reshape(-1)
    y = np.empty(x.size, dtype=np.float64)
    lib().oracle_gelu(_ptr(x), x.size, _ptr(y))
    return y.reshape(np.shape(x_bits))


# ---- INT8 query/key quantization for attention scores ----------------------
#
# FastH3 Trim (comfyui-wiki news), "How fast it runs": on the RTX 4090 the
# FP8 path quantizes the query and the key to INT8 for the score computation.
# The pages fix neither the granularity nor the rounding; this oracle takes the
# plainest reading: one symmetric scale per row (one token of one head),
#   s = fp32(amax_row / 127)                      (IEEE single division)
#   q = clamp(rne(fp32(x / s)), -127, 127)        (IEEE single division, then
#                                                  round half to even)
# with s = 0 and q = 0 for an all-zero row.  The decisions are taken in FP32:
# the method keeps one scale per row and multiplies it back into the integer
# scores, so that scale is a stored FP32 number, and the quotient that decides
# each code is the quotient by that stored number, correctly rounded to FP32
# like the scale itself (numpy's float32 division is the IEEE correctly
# rounded one).

def quantize_int8_rows(x_bits: np.ndarray):
    """BF16 bits [rows, d] -> (int8 [rows, d], float32 scales [rows])."""
    x = (x_bits.astype(np.uint32) << 16).view(np.float32).reshape(x_bits.shape)
    amax = np.abs(x).max(axis=1).astype(np.float32)
    s = (amax / np.float32(127.0)).astype(np.float32)
    q = np.zeros(x.shape, dtype=np.int8)
    nz = s > 0
    with np.errstate(invalid="ignore", divide="ignore"):
        r = (x[nz] / s[nz, None]).astype(np.float32)
    q[nz] = np.clip(np.rint(r), -127, 127).astype(np.int8)
    return q, s


def int8_scores(q8: np.ndarray, q_scales: np.ndarray, k8: np.ndarray, k_scales: np.ndarray,
                sm_scale: float) -> np.ndarray:
    """S[h, i, j] = sm_scale * s_q[h, i] * s_k[h, j] * sum_d q[h, i, d] k[h, j, d] in binary64
    (the integer sums are exact); q8 [H, Tq, d], k8 [H, Tk, d], scales [H, T]."""
    acc = np.einsum("hid,hjd->hij", q8.astype(np.int64), k8.astype(np.int64))
    return (float(sm_scale) * q_scales.astype(np.float64)[:, :, None] * k_scales.astype(np.float64)[:, None, :]
            * acc.astype(np.float64))


def int8_scores_tolerance(s_ref: np.ndarray) -> np.ndarray:
    """Allowed |S - S_ref| for S = (float(acc) * (s_q * sm_scale)) * s_k evaluated in FP32: at
    most four roundings separate it from the exact product (the conversion of acc, exact while
    |acc| < 2^24, and the three multiplies), each within 2^-24 relative, so |S - S_ref| <=
    ((1 + 2^-24)^4 - 1) |S_ref| < 4 * 2^-24 * (1 + 2^-20) |S_ref|; the factor also covers
    the binary64 rounding of S_ref.  The 1e-30 absolute term covers FP32 underflow."""
    return 4.0 * 2.0 ** -24 * (1.0 + 2.0 ** -20) * np.abs(s_ref) + 1e-30


# ---- AdaLN timestep conditioning through a shared low-rank basis -------------------
# FastH3 Trim (comfyui-wiki news), "What Trim changes": AdaLN maps the 2,688-wide
# time embedding to six modulation vectors per block; Trim replaces the per-block
# projections with one shared 2,688 -> 16 basis followed by a small projection per
# block, both stored in FP16.  Reading: the two maps are linear,
#   code[b, j]       = sum_k basis[j, k] * e[b, k]                  (r = 16 values)
#   mod[l, b, i]     = sum_j proj[l, i, j] * code[b, j] + bias[l, i] (6 * 2688 values)
# with BF16 embeddings, FP16 weights and exact (binary64) arithmetic here.

def f16_to_f64(bits: np.ndarray) -> np.ndarray:
    """IEEE half bits -> float64 (exact)."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def adaln_code(e_bits: np.ndarray, basis_bits: np.ndarray) -> np.ndarray:
    """code [bt, r] = e [bt, d] (BF16 bits) times basis^T, basis [r, d] (FP16 bits), in binary64."""
    e = (np.asarray(e_bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)
    return e @ f16_to_f64(basis_bits).T


def adaln_modulation(code: np.ndarray, proj_bits: np.ndarray, bias_bits) -> np.ndarray:
    """mod [L, bt, n] = proj [L, n, r] (FP16 bits) applied to code [bt, r], plus bias [L, n] (FP16 bits)."""
    proj = f16_to_f64(proj_bits)
    out = np.einsum("lir,br->lbi", proj, code)
    if bias_bits is not None:
        out = out + f16_to_f64(bias_bits)[:, None, :]
    return out


def adaln_tolerance(e_bits, basis_bits, proj_bits, bias_bits) -> np.ndarray:
    """Worst-case bound for FP32 evaluation of the two maps in any summation order
    (Higham's dot-product bound, gamma_n = n u / (1 - n u), u = 2^-24, applied to the
    code and then to the projection):  |err| <= (gamma_d + gamma_{r+1} + gamma_d
    gamma_{r+1}) * M, where M is the same expression evaluated on absolute values."""
    e = np.abs((np.asarray(e_bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64))
    code_abs = e @ np.abs(f16_to_f64(basis_bits)).T
    m = np.einsum("lir,br->lbi", np.abs(f16_to_f64(proj_bits)), code_abs)
    if bias_bits is not None:
        m = m + np.abs(f16_to_f64(bias_bits))[:, None, :]
    u = 2.0 ** -24
    d, r = np.shape(e_bits)[1], np.shape(basis_bits)[0]
    g1 = d * u / (1 - d * u)
    g2 = (r + 1) * u / (1 - (r + 1) * u)
    return (g1 + g2 + g1 * g2) * m * (1 + 1e-12) + 1e-37
