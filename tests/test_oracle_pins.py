"""Pins of the CPU oracle against facts that do not come from the oracle itself.

- hand-worked blocks (tests/golden/nvfp4_block_cases.json);
- torch's float8_e4m3fn conversions (an independent library) for the E4M3 codec;
- exact rational brute force (fractions.Fraction, nearest-by-distance search)
  for block scales, element codes, the global-scale rule and small GEMMs;
- invariants: sign symmetry, idempotence, power-of-two scaling, clip counts
  of calibrated versus uncalibrated scales (FastH3 thread digest, farwalk.ai,
  tweet 6/8: uncalibrated FP4 scales clip, calibrated ones keep the large
  activations intact).
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import synthetic as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "nvfp4_block_cases.json")
E2M1_GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def bf16_bits_of(values):
    t = torch.tensor(values, dtype=torch.float32).to(torch.bfloat16)
    assert torch.equal(t.to(torch.float32), torch.tensor(values, dtype=torch.float32)), "not exact in BF16"
    return t.view(torch.int16).numpy().view(np.uint16)


def e4m3_values_by_torch():
    return torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()


# --------------------------------------------------------------------------
# Hand-worked cases
# --------------------------------------------------------------------------

def golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", golden_cases(), ids=lambda c: c["name"][:40])
def test_golden_block(oracle_mod, case):
    x = bf16_bits_of(case["x"]).reshape(1, 16)
    codes, scales, clip = oracle_mod.quantize(x, case["sg"])
    assert scales.tobytes().hex() == case["scale"]
    assert codes.tobytes().hex() == case["codes"]
    assert clip == case["clip"]


def test_golden_blocks_in_one_matrix(oracle_mod):
    """Rows and blocks are indexed independently: stacking the same-sg cases as
    blocks of one row and as rows of one matrix gives the same bytes."""
    cases = [c for c in golden_cases() if c["sg"] == 1.0]
    row = bf16_bits_of(sum((c["x"] for c in cases), [])).reshape(1, -1)
    codes, scales, clip = oracle_mod.quantize(row, 1.0)
    assert scales.tobytes().hex() == "".join(c["scale"] for c in cases)
    assert codes.tobytes().hex() == "".join(c["codes"] for c in cases)
    assert clip == sum(c["clip"] for c in cases)
    mat = np.concatenate([bf16_bits_of(c["x"]).reshape(1, 16) for c in cases])
    codes2, scales2, _ = oracle_mod.quantize(mat, 1.0)
    assert codes2.tobytes() == codes.tobytes() and scales2.tobytes() == scales.tobytes()


# --------------------------------------------------------------------------
# Element codecs
# --------------------------------------------------------------------------

def test_e2m1_decode_grid(oracle_mod):
    assert [oracle_mod.e2m1_value(c) for c in range(8)] == E2M1_GRID
    assert [oracle_mod.e2m1_value(c | 8) for c in range(8)] == [-v for v in E2M1_GRID]
    assert math.copysign(1.0, oracle_mod.e2m1_value(8)) == -1.0


def test_e2m1_encode_ties_and_saturation(oracle_mod):
    expect = {0.0: 0, 0.25: 0, 0.5: 1, 0.75: 2, 1.0: 2, 1.25: 2, 1.5: 3, 1.75: 4, 2.0: 4,
              2.5: 4, 3.0: 5, 3.5: 6, 4.0: 6, 5.0: 6, 6.0: 7, 6.5: 7, 1e30: 7,
              0.2499: 0, 0.2501: 1, 0.7499: 1, 4.9999: 6, 5.0001: 7}
    for r, c in expect.items():
        assert oracle_mod.e2m1_rne_sat(r) == c, r


def test_e4m3_decode_all_bytes_against_torch(oracle_mod):
    ref = e4m3_values_by_torch()
    for b in range(256):
        v = oracle_mod.e4m3_value(b)
        if math.isnan(ref[b]):
            assert math.isnan(v), b
        else:
            assert v == ref[b] and math.copysign(1, v) == math.copysign(1, ref[b]), b
    assert oracle_mod.e4m3_value(0x7E) == 448.0 and oracle_mod.e4m3_value(0x01) == 2.0 ** -9


def test_e4m3_encode_against_torch(oracle_mod):
    ref = e4m3_values_by_torch()[:0x7F]
    mids = (ref[:-1] + ref[1:]) / 2
    rng = np.random.default_rng(7)
    qs = np.concatenate([ref, mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9),
                         rng.uniform(0, 500, 3000), np.exp(rng.uniform(np.log(1e-5), np.log(600), 3000)),
                         [448, 460, 463.99, 464, 500, 1e6]]).astype(np.float32)
    t = torch.from_numpy(qs).clamp(max=448.0).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle_mod.e4m3_rne_sat(float(q)) for q in qs])
    np.testing.assert_array_equal(got, t)


# --------------------------------------------------------------------------
# Exact rational brute force
# --------------------------------------------------------------------------

def nearest_even(q: Fraction, grid, max_code):
    """Nearest grid value by exact distance, ties to the even code; q beyond the
    top saturates."""
    best = None
    for c in range(max_code + 1):
        d = abs(q - grid[c])
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
            best = (d, c)
    return best[1]


def brute_quantize_block(xs, sg):
    e4 = [Fraction(v) for v in e4m3_values_by_torch()[:0x7F]]
    e2 = [Fraction(v) for v in E2M1_GRID]
    sgf = Fraction(sg)
    amax = max(abs(Fraction(v)) for v in xs)
    sc = nearest_even(amax / (6 * sgf), e4, 0x7E)
    Sv = e4[sc]
    codes = []
    for v in xs:
        sign = 8 if math.copysign(1.0, v) < 0 else 0
        codes.append(sign if Sv == 0 else sign | nearest_even(abs(Fraction(v)) / (Sv * sgf), e2, 7))
    clip = sum(1 for v in xs if abs(Fraction(v)) > 2688 * sgf)
    return sc, codes, clip


def unpack(codes_row):
    out = []
    for b in codes_row:
        out += [int(b) & 15, int(b) >> 4]
    return out


@pytest.mark.parametrize("seed", range(6))
def test_quantize_matches_rational_brute_force(oracle_mod, seed):
    rng = np.random.default_rng(seed)
    # blocks with assorted magnitudes, including tiny ones (subnormal scales)
    nblk = 48
    mags = np.exp(rng.uniform(np.log(1e-4), np.log(5e3), nblk))
    x = S.to_bf16_bits(rng.standard_normal((nblk, 16)) * mags[:, None])
    sg = float(np.float32(np.exp(rng.uniform(np.log(1e-3), np.log(4.0)))))
    codes, scales, clip = oracle_mod.quantize(x.reshape(1, -1), sg)
    xf = S.bf16_to_f32(x).astype(np.float64)
    tot = 0
    for b in range(nblk):
        sc, cs, cl = brute_quantize_block(list(xf[b]), sg)
        assert scales[0, b] == sc
        assert unpack(codes[0, 8 * b:8 * b + 8]) == cs
        tot += cl
    assert clip == tot


def test_quantize_brute_force_at_exact_ties(oracle_mod):
    """Blocks built so every element sits exactly on an E2M1 midpoint for its
    block scale, at non-power-of-two scales (the hardest rounding cases)."""
    rng = np.random.default_rng(11)
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    rows = []
    for sc_val in [1.125, 1.25, 1.375, 1.5, 1.625, 1.75, 1.875, 0.75, 3.0, 5.0, 13.0]:
        amax = 6 * sc_val                       # q = sc_val exactly -> S = sc_val
        vals = [amax] + [m * sc_val * (-1) ** i for i, m in enumerate(rng.choice(mids, 15))]
        rows.append(vals)
    xs = np.array(rows)
    x = S.to_bf16_bits(xs)
    assert np.array_equal(S.bf16_to_f32(x).astype(np.float64), xs)
    codes, scales, _ = oracle_mod.quantize(x, 1.0)
    for r in range(len(rows)):
        sc, cs, _ = brute_quantize_block(rows[r], 1.0)
        assert scales[r, 0] == sc and unpack(codes[r]) == cs


# --------------------------------------------------------------------------
# Invariants
# --------------------------------------------------------------------------

def test_sign_symmetry(oracle_mod):
    x = S.random_bf16(("pin", "sign"), (8, 256), 3.0)
    sg = 0.0123
    c1, s1, k1 = oracle_mod.quantize(x, sg)
    c2, s2, k2 = oracle_mod.quantize(x ^ np.uint16(0x8000), sg)
    np.testing.assert_array_equal(s1, s2)
    np.testing.assert_array_equal(c1 ^ np.uint8(0x88), c2)
    assert k1 == k2


def test_power_of_two_scaling(oracle_mod):
    x = S.random_bf16(("pin", "pow2"), (8, 256), 2.0)
    xf = S.bf16_to_f32(x).astype(np.float64)
    c1, s1, _ = oracle_mod.quantize(x, 0.01)
    c2, s2, _ = oracle_mod.quantize(S.to_bf16_bits(xf * 4.0), 0.04)
    np.testing.assert_array_equal(c1, c2)
    np.testing.assert_array_equal(s1, s2)


def test_idempotence(oracle_mod):
    """Re-quantizing the dequantized tensor (exact in BF16 when s_g is a power
    of two) reproduces codes and scales for blocks with normal-range scales."""
    x = S.random_bf16(("pin", "idem"), (16, 256), 1.0)
    sg = 2.0 ** -9
    codes, scales, _ = oracle_mod.quantize(x, sg)
    e4 = e4m3_values_by_torch()
    deq = np.empty((16, 256))
    for r in range(16):
        cs = unpack(codes[r])
        for k in range(256):
            deq[r, k] = math.copysign(E2M1_GRID[cs[k] & 7], -1.0 if cs[k] & 8 else 1.0) * e4[scales[r, k // 16]] * sg
    assert (scales >= 0x08).all()               # normal E4M3 scales only
    x2 = S.to_bf16_bits(deq)
    assert np.array_equal(S.bf16_to_f32(x2).astype(np.float64), deq)
    codes2, scales2, _ = oracle_mod.quantize(x2, sg)
    np.testing.assert_array_equal(scales2, scales)
    np.testing.assert_array_equal(codes2, codes)


# --------------------------------------------------------------------------
# Global scale rule and amax
# --------------------------------------------------------------------------

def test_scale_from_amax_special_values(oracle_mod):
    assert oracle_mod.scale_from_amax(2688.0) == 1.0
    assert oracle_mod.scale_from_amax(1344.0) == 0.5
    assert oracle_mod.scale_from_amax(0.0) == 1.0


def test_scale_from_amax_is_minimal(oracle_mod):
    rng = np.random.default_rng(3)
    amaxes = np.concatenate([np.exp(rng.uniform(np.log(1e-6), np.log(1e5), 300)), [1096.0, 4.5, 0.0625]])
    for a in S.bf16_to_f32(S.to_bf16_bits(amaxes)):
        s = np.float32(oracle_mod.scale_from_amax(float(a)))
        prev = np.nextafter(s, np.float32(0))
        assert Fraction(float(s)) * 2688 >= Fraction(float(a))
        assert Fraction(float(prev)) * 2688 < Fraction(float(a))


def test_amax(oracle_mod):
    x = S.random_bf16(("pin", "amax"), (33, 77), 5.0)
    assert oracle_mod.amax(x) == float(np.abs(S.bf16_to_f32(x)).max())


def test_calibrated_scale_never_clips_and_uncalibrated_clips_outliers(oracle_mod):
    """The tiny workload: 16 calibration batches of 128 tokens with 0.1% outliers
    at 137 times the clip limit.  The calibrated scale clips nothing; a scale
    set from the non-outlier amax clips exactly the injected outliers."""
    layer = S.workloads()["tiny"][0]
    calib = S.activation_batches(layer, 0, layer.n_calib)
    sg = oracle_mod.scale_from_amax(oracle_mod.amax(calib))
    x = S.activations(layer)
    _, _, clip = oracle_mod.quantize(x, sg)
    assert clip == 0
    body = S.activation_batches(layer, 0, 1, uncalibrated_body=True)
    pos = S.outlier_positions(layer, 0)
    xb = x.reshape(-1).copy()
    assert np.array_equal(np.delete(xb, pos), np.delete(body.reshape(-1), pos))
    sg_unc = oracle_mod.scale_from_amax(oracle_mod.amax(np.delete(xb, pos)))
    _, _, clip_unc = oracle_mod.quantize(x, sg_unc)
    assert clip_unc == layer.outliers_per_batch() == 33


# --------------------------------------------------------------------------
# Tensor-core scale layout
# --------------------------------------------------------------------------

def test_tiled_scale_layout_worked_positions(oracle_mod):
    off = oracle_mod.tiled_scale_offsets(256, 512)        # 32 scale columns -> 8 K-atoms
    assert off[0, 0] == 0 and off[0, 1] == 1 and off[0, 3] == 3
    assert off[1, 0] == 16 and off[31, 0] == 31 * 16
    assert off[32, 0] == 4 and off[64, 2] == 10 and off[127, 3] == 31 * 16 + 12 + 3
    assert off[0, 4] == 512 and off[0, 31] == 7 * 512 + 3
    assert off[128, 0] == 8 * 512
    flat = np.sort(off.reshape(-1))
    np.testing.assert_array_equal(flat, np.arange(256 * 32))
    assert oracle_mod.tiled_scales_bytes(100, 48) == 128 * 4


# --------------------------------------------------------------------------
# Linear layer
# --------------------------------------------------------------------------

def random_quantized(rng, rows, K, max_scale_code=0x50):
    codes = rng.integers(0, 256, (rows, K // 2), dtype=np.uint8)
    scales = rng.integers(0, max_scale_code, (rows, K // 16), dtype=np.uint8)
    return codes, scales


def dequant_fraction(codes, scales, r, k):
    e4 = e4m3_values_by_torch()
    b = int(codes[r, k // 2])
    c = (b & 15) if k % 2 == 0 else (b >> 4)
    v = Fraction(E2M1_GRID[c & 7]) * (-1 if c & 8 else 1)
    return v * Fraction(float(e4[scales[r, k // 16]]))


@pytest.mark.parametrize("shape", [(3, 16, 5), (8, 32, 16), (17, 48, 9)])
def test_linear_matches_rational_brute_force(oracle_mod, shape):
    M, K, N = shape
    rng = np.random.default_rng(M * 1000 + K)
    ac, asc = random_quantized(rng, M, K)
    wc, wsc = random_quantized(rng, N, K)
    bias = S.random_bf16(("pin", "bias", M), (N,), 0.5)
    ag, wg = 0.37109375, 0.0013427734375
    y, mag = oracle_mod.linear(ac, asc, ag, wc, wsc, wg, bias)
    for m in range(M):
        for n in range(N):
            prods = [dequant_fraction(ac, asc, m, k) * dequant_fraction(wc, wsc, n, k) for k in range(K)]
            exact = Fraction(ag) * Fraction(wg) * sum(prods) + Fraction(float(S.bf16_to_f32(bias[n:n + 1])[0]))
            exact_mag = abs(Fraction(ag) * Fraction(wg)) * sum(abs(p) for p in prods)
            assert abs(Fraction(y[m, n]) - exact) <= Fraction(2) ** -50 * (abs(exact) + exact_mag + 1)
            assert abs(Fraction(mag[m, n]) - exact_mag) <= Fraction(2) ** -50 * (exact_mag + 1)


def test_linear_unit_scales_is_integer_matmul(oracle_mod):
    """All block scales 1.0 (0x38) and unit global scales: y = decoded codes
    matmul (torch float64) plus bias."""
    rng = np.random.default_rng(5)
    M, K, N = 20, 64, 24
    ac = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    wc = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    asc = np.full((M, K // 16), 0x38, np.uint8)
    wsc = np.full((N, K // 16), 0x38, np.uint8)
    lut = np.array(E2M1_GRID + [-v for v in E2M1_GRID])
    A = np.stack([lut[ac & 15], lut[ac >> 4]], axis=-1).reshape(M, K)
    W = np.stack([lut[wc & 15], lut[wc >> 4]], axis=-1).reshape(N, K)
    ref = (torch.from_numpy(A) @ torch.from_numpy(W).T).numpy()
    y, mag = oracle_mod.linear(ac, asc, 1.0, wc, wsc, 1.0, None)
    np.testing.assert_array_equal(y, ref)
    np.testing.assert_array_equal(mag, (torch.from_numpy(np.abs(A)) @ torch.from_numpy(np.abs(W)).T).numpy())


def test_linear_one_hot(oracle_mod):
    K, N = 64, 3
    ac = np.zeros((1, K // 2), np.uint8)
    ac[0, 21] = 0x70                       # element 43 = code 7 (6.0)
    asc = np.zeros((1, K // 16), np.uint8)
    asc[0, 2] = 0x40                       # block 2 scale = 2.0
    wc = np.zeros((N, K // 2), np.uint8)
    wc[1, 21] = 0xD0                       # W[1, 43] = code 13 (-3.0)
    wsc = np.full((N, K // 16), 0x30, np.uint8)   # 0.5
    bias = np.array([0x3F80, 0, 0xBF80], np.uint16)   # 1, 0, -1
    y, mag = oracle_mod.linear(ac, asc, 0.25, wc, wsc, 4.0, bias)
    np.testing.assert_array_equal(y[0], [1.0, 6.0 * 2.0 * -3.0 * 0.5, -1.0])
    np.testing.assert_array_equal(mag[0], [0.0, 18.0, 0.0])


def test_gelu(oracle_mod):
    """GELU(x) = x Phi(x): tabulated normal CDF values, the identity
    GELU(x) - GELU(-x) = x, and the asymptotic tail series
    x Phi(x) ~ -phi(x) (1 - 1/x^2 + 3/x^4 - 15/x^6 + 105/x^8) for x -> -inf."""
    x = np.array([0x0000, 0x3F80, 0xBF80, 0x4000], np.uint16)   # 0, 1, -1, 2
    y = oracle_mod.gelu(x)
    ref = [0.0, 0.8413447460685429, -0.15865525393145707, 2 * 0.9772498680518208]
    np.testing.assert_allclose(y, ref, rtol=1e-15, atol=0)
    v = S.random_bf16(("pin", "gelu"), (1000,), 3.0)
    d = oracle_mod.gelu(v) - oracle_mod.gelu(v ^ np.uint16(0x8000))
    np.testing.assert_allclose(d, S.bf16_to_f32(v).astype(np.float64), rtol=1e-14, atol=1e-300)
    for xv in [-8.0, -9.0, -10.0, -12.0]:
        series = 1 - 1 / xv**2 + 3 / xv**4 - 15 / xv**6 + 105 / xv**8
        asym = -math.exp(-xv * xv / 2) / math.sqrt(2 * math.pi) * series
        got = oracle_mod.gelu(S.to_bf16_bits(np.array([xv])))[0]
        bound = 945 / xv**10 * 1.01     # the next term of the alternating series
        assert abs(got - asym) <= abs(asym) * bound, (xv, got, asym)


def test_clip_count_at_the_limit_and_by_brute_force(oracle_mod):
    """clip_count counts |x| > 2688 s_g exactly: an element equal to the limit
    is not clipped, the next BF16 above it is, in both signs; on random wide-
    range inputs it equals a rational count and quantize()'s clip count."""
    sg = 1.0 / 1024                       # limit 2688 / 1024 = 2.625, a BF16 value
    lim = S.to_bf16_bits(np.array([2.625]))[0]
    above = np.uint16(lim + 1)            # next BF16 magnitude up
    below = np.uint16(lim - 1)
    row = np.array([lim, above, below, lim | 0x8000, above | 0x8000, 0, 0x8000, below | 0x8000] * 2, dtype=np.uint16)
    assert oracle_mod.clip_count(row, sg) == 4
    assert oracle_mod.quantize(row.reshape(1, -1), sg)[2] == 4
    rng = np.random.default_rng(5)
    x = S.to_bf16_bits(rng.standard_normal((64, 128)) * np.exp(rng.uniform(-3, 3, (64, 1))))
    for sg in (1e-3, 2.0 ** -12, float(np.float32(0.0037))):
        want = sum(1 for v in S.bf16_to_f32(x).reshape(-1) if abs(Fraction(float(v))) > 2688 * Fraction(sg))
        assert oracle_mod.clip_count(x, sg) == want == oracle_mod.quantize(x, sg)[2]
