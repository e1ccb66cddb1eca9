"""Pins of the oracle's INT8 query/key quantization and score computation
(reading R13: per-row symmetric scale s = fp32(amax / 127), codes
clamp(rne(fp32(x / s)), -127, 127)), against definitions computed another way."""
from fractions import Fraction

import numpy as np

import oracle
import synthetic as S


def _f32(v):
    return float(np.float32(v))


def test_int8_rows_hand_worked():
    # Row with amax 127: s = 1 exactly, codes are the values rounded half to even.
    vals = [127.0, -127.0, 0.5, 1.5, 2.5, -2.5, 3.0, 0.0]
    x = S.to_bf16_bits(np.array(vals, dtype=np.float64)).reshape(1, -1)
    q, s = oracle.quantize_int8_rows(x)
    assert s[0] == np.float32(1.0)
    assert q.tolist() == [[127, -127, 0, 2, 2, -2, 3, 0]]


def test_int8_rows_zero_row_and_amax_maps_to_127():
    x = S.to_bf16_bits(np.array([[0.0] * 8, [0.0, 0.0, -3.0, 1.0, 2.0, 0.0, 0.0, 0.0]]))
    q, s = oracle.quantize_int8_rows(x)
    assert s[0] == 0 and (q[0] == 0).all()
    assert s[1] == np.float32(np.float32(3.0) / np.float32(127.0))
    assert q[1, 2] == -127 and abs(int(q[1, 3])) == 42  # 1 / (3/127) = 42.33


def test_int8_rows_against_per_element_definition():
    """Element by element with Python floats rounded to binary32 at each step."""
    rng = np.random.default_rng(3)
    x = S.to_bf16_bits(rng.standard_normal((40, 64)) * np.exp(rng.uniform(-8, 8, (40, 1))))
    q, s = oracle.quantize_int8_rows(x)
    xv = S.bf16_to_f32(x).astype(np.float64)
    for i in range(x.shape[0]):
        amax = max(abs(v) for v in xv[i])
        si = _f32(np.float32(amax) / np.float32(127.0))
        assert s[i] == np.float32(si)
        for j in range(x.shape[1]):
            r = _f32(np.float32(xv[i, j]) / np.float32(si))
            fl = np.floor(r)
            d = r - fl
            k = fl + 1 if d > 0.5 or (d == 0.5 and fl % 2 == 1) else fl  # half to even
            assert q[i, j] == int(max(-127, min(127, k)))


def test_int8_rows_codes_within_half_step():
    """|x - q s| <= s (1/2 + 2^-17) for every element: the code rounds the FP32
    quotient x / s, which lies within half an ulp (<= 2^-17 below 128) of the exact one."""
    rng = np.random.default_rng(4)
    x = S.to_bf16_bits(rng.standard_normal((64, 128)) * 3.0)
    q, s = oracle.quantize_int8_rows(x)
    xv = S.bf16_to_f32(x).astype(np.float64)
    err = np.abs(xv - q.astype(np.float64) * s[:, None].astype(np.float64))
    assert (err <= s[:, None] * (0.5 + 2.0 ** -17)).all()
    assert (np.abs(q) <= 127).all()


def test_int8_scores_brute_force():
    """Exact rationals on a tiny case: the binary64 result is the exact product rounded once."""
    rng = np.random.default_rng(5)
    q8 = rng.integers(-127, 128, (2, 3, 32)).astype(np.int8)
    k8 = rng.integers(-127, 128, (2, 4, 32)).astype(np.int8)
    qs = rng.uniform(0.001, 0.1, (2, 3)).astype(np.float32)
    ks = rng.uniform(0.001, 0.1, (2, 4)).astype(np.float32)
    out = oracle.int8_scores(q8, qs, k8, ks, 0.125)
    for h in range(2):
        for i in range(3):
            for j in range(4):
                acc = sum(int(a) * int(b) for a, b in zip(q8[h, i], k8[h, j]))
                exact = Fraction(1, 8) * Fraction(float(qs[h, i])) * Fraction(float(ks[h, j])) * acc
                assert abs(Fraction(out[h, i, j]) - exact) <= abs(exact) * Fraction(1, 2 ** 50)


def test_int8_scores_dequantized_close_to_float_product():
    """Scores of quantized rows approximate the float scores within the quantization error."""
    rng = np.random.default_rng(6)
    xq = S.to_bf16_bits(rng.standard_normal((1, 16, 128)).reshape(16, 128))
    xk = S.to_bf16_bits(rng.standard_normal((1, 20, 128)).reshape(20, 128))
    q, qs = oracle.quantize_int8_rows(xq)
    k, ks = oracle.quantize_int8_rows(xk)
    s = oracle.int8_scores(q[None], qs[None], k[None], ks[None], 1.0)[0]
    ref = S.bf16_to_f32(xq).astype(np.float64) @ S.bf16_to_f32(xk).astype(np.float64).T
    bound = 128 * (np.abs(S.bf16_to_f32(xq)).max() * ks.max() + np.abs(S.bf16_to_f32(xk)).max() * qs.max())
    assert np.abs(s - ref).max() <= bound


def test_score_tolerance_covers_fp32_evaluation_and_no_more():
    """The four-rounding bound: the scores evaluated in FP32 in the stated order
    (float(acc) * (s_q * sm_scale)) * s_k -- here with numpy's float32, including
    sums past 2^24 whose conversion rounds -- lie within the tolerance of the
    binary64 scores, and values five FP32 ulps away do not."""
    rng = np.random.default_rng(3)
    d = 2688
    q8 = rng.integers(-127, 128, size=(1, 24, d)).astype(np.int8)
    q8[0, :4] = 127                                        # |acc| up to 127^2 d > 2^24: the conversion rounds
    k8 = rng.integers(-127, 128, size=(1, 40, d)).astype(np.int8)
    k8[0, :4] = 127
    qs = rng.uniform(1e-3, 2.0, size=(1, 24)).astype(np.float32)
    ks = rng.uniform(1e-3, 2.0, size=(1, 40)).astype(np.float32)
    sm = np.float32(1.0 / np.sqrt(128.0))
    ref = oracle.int8_scores(q8, qs, k8, ks, float(sm))
    acc = np.einsum("hid,hjd->hij", q8.astype(np.int64), k8.astype(np.int64))
    assert np.abs(acc).max() > 2 ** 24
    s32 = (acc.astype(np.float32) * (qs * sm)[:, :, None]) * ks[:, None, :]
    tol = oracle.int8_scores_tolerance(ref)
    assert (np.abs(s32.astype(np.float64) - ref) <= tol).all()
    far = ref * (1.0 + 5 * 2.0 ** -24) + np.sign(ref) * 1e-29
    big = np.abs(ref) > 1e-20
    assert (np.abs(far - ref)[big] > tol[big]).all()
