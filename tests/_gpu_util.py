"""Helpers shared by the GPU parity tests: move seeded BF16 bits to the GPU,
run the library through its binding, and compare with the oracle."""
import numpy as np
import torch

import oracle
import synthetic as S


def fh():
    import nvfp4_quantized_linear_fh_b200 as m
    return m


def to_dev(bits: np.ndarray, ldx: int | None = None) -> torch.Tensor:
    """uint16 BF16 bits [M, K] -> CUDA bfloat16 tensor (optionally inside a wider row stride)."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    t = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    if ldx is not None and bits.ndim == 2 and ldx != bits.shape[1]:
        wide = torch.zeros((bits.shape[0], ldx), dtype=torch.bfloat16, device="cuda")
        wide[:, :bits.shape[1]] = t
        return wide[:, :bits.shape[1]]
    return t


def gpu_quantize(x_dev: torch.Tensor, sg: float, layout: int):
    m = fh()
    M, K = x_dev.shape
    codes, scales = m.empty_quantized(M, K, layout=layout)
    scales.fill_(0xA5)  # poison: every byte the layout defines must be written
    clip = torch.zeros(1, dtype=torch.int64, device="cuda")
    m.fh_quantize_act(x_dev, sg, codes, scales, clip, layout)
    return codes, scales, clip


def check_quantize(x_bits: np.ndarray, sg: float, layout: int, ldx: int | None = None):
    """Bit-exact comparison of codes, scales and clip count with the oracle."""
    m = fh()
    M, K = x_bits.shape
    oc, osc, ocl = oracle.quantize(x_bits, sg)
    codes, scales, clip = gpu_quantize(to_dev(x_bits, ldx), sg, layout)
    torch.cuda.synchronize()
    gc = codes.cpu().numpy()
    gs = scales.cpu().numpy()
    bad = np.argwhere(gc != oc)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first at {bad[:5].tolist()}"
    if layout == m.FH_SCALES_ROWMAJOR:
        np.testing.assert_array_equal(gs[:M * (K // 16)].reshape(M, K // 16), osc)
    else:
        off = oracle.tiled_scale_offsets(M, K)
        np.testing.assert_array_equal(gs[off], osc)
        rest = np.ones(gs.size, dtype=bool)
        rest[off.reshape(-1)] = False
        assert (gs[rest] == 0).all(), "padding scales must be zero"
    assert int(clip.item()) == ocl
    return ocl


def quantize_tiled(x_dev: torch.Tensor, sg: float):
    m = fh()
    codes, scales, clip = gpu_quantize(x_dev, sg, m.FH_SCALES_MMA_TILED)
    return codes, scales, clip


def sample_rows(M: int, n: int, seed: int = 0) -> np.ndarray:
    fixed = [0, 1, 31, 32, 127, 128, M // 2, M - 2, M - 1]
    rng = np.random.default_rng(seed)
    extra = rng.choice(M, size=max(0, min(n, M) - len(fixed)), replace=False)
    return np.unique(np.clip(np.concatenate([fixed, extra]), 0, M - 1)).astype(np.int64)


def check_linear(y_dev: torch.Tensor, a_bits: np.ndarray, a_g: float, w_bits: np.ndarray, w_g: float,
                 bias_bits, rows=None):
    """GEMM output within |y - y_ref| <= 2^-8 |y_ref| + 1e-5 sum|a b| on the given rows
    (the oracle quantizes the same BF16 inputs itself)."""
    ac, asc, _ = oracle.quantize(a_bits if rows is None else a_bits[rows], a_g)
    wc, wsc, _ = oracle.quantize(w_bits, w_g)
    y_ref, mag = oracle.linear(ac, asc, a_g, wc, wsc, w_g, bias_bits)
    y = S.bf16_to_f32(y_dev.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)
    if rows is not None:
        y = y[rows]
    err = np.abs(y - y_ref)
    tol = oracle.linear_tolerance(y_ref, mag)
    worst = np.unravel_index(np.argmax(err - tol), err.shape)
    assert (err <= tol).all(), (f"{int((err > tol).sum())} of {err.size} outputs out of tolerance; worst at "
                                f"{worst}: y={y[worst]}, ref={y_ref[worst]}, tol={tol[worst]}")
    return float((err / np.maximum(tol, 1e-300)).max())


def tile_rows(M: int, salt: int = 0) -> np.ndarray:
    """One row in every 128-row tile of an M-row output (its place inside the
    tile moves from tile to tile, so every TMEM lane quadrant and both CTAs of
    a 256-row pair tile are visited), plus the rows at the edges of the
    matrix, of the 256-row pair tiles and of the 32-row quadrants."""
    tiles = np.arange((M + 127) // 128)
    rows = tiles * 128 + (tiles * 37 + salt * 11 + 5) % 128
    edges = [0, 1, 31, 32, 63, 64, 95, 96, 127, 128, 255, 256, M - 257, M - 256, M - 129, M - 128, M - 2, M - 1]
    rows = np.concatenate([rows, np.array(edges)])
    return np.unique(rows[(rows >= 0) & (rows < M)]).astype(np.int64)


def bits_of(t: torch.Tensor) -> np.ndarray:
    """The uint16 BF16 bits of a CUDA bfloat16 (or int16) tensor, on the host."""
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def check_quantized(codes: torch.Tensor, scales: torch.Tensor, clip: int, x_bits: np.ndarray, sg: float):
    """Bit-exact comparison of a tensor-core-layout quantization the GPU already
    made (codes, scales, clip count) with the oracle's quantization of x_bits."""
    M, K = x_bits.shape
    oc, osc, ocl = oracle.quantize(x_bits, sg)
    gc = codes.cpu().numpy()
    bad = np.argwhere(gc != oc)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first at {bad[:5].tolist()}"
    gs = scales.cpu().numpy()
    off = oracle.tiled_scale_offsets(M, K)
    np.testing.assert_array_equal(gs[off], osc)
    rest = np.ones(gs.size, dtype=bool)
    rest[off.reshape(-1)] = False
    assert (gs[rest] == 0).all(), "padding scales must be zero"
    assert clip == ocl
    return ocl
