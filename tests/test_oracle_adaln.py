"""Pins of the oracle's AdaLN basis projection (FastH3 Trim, comfyui-wiki news, "What
Trim changes": a shared 2,688 -> 16 basis plus a small per-block projection, in FP16):
exact rational brute force, closed forms (one-hot and zero embeddings, integer data),
the dense projection the factorization stands for, and the FP32 error bound."""
from fractions import Fraction

import numpy as np

import oracle
import synthetic as S


def _bf16(x):
    return S.to_bf16_bits(np.asarray(x, dtype=np.float64))


def _f16(x):
    return S.to_f16_bits(np.asarray(x, dtype=np.float64))


def _vals_bf16(bits):
    return [[Fraction(float(v)) for v in row] for row in S.bf16_to_f32(bits).astype(np.float64)]


def _vals_f16(bits):
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def test_brute_force_rationals():
    """Tiny case in exact rationals: the oracle differs only by binary64 rounding."""
    rng = np.random.default_rng(11)
    L, n, d, r, bt = 2, 5, 8, 3, 2
    e = _bf16(rng.standard_normal((bt, d)))
    basis = _f16(rng.standard_normal((r, d)) / 3)
    proj = _f16(rng.standard_normal((L, n, r)) / 5)
    bias = _f16(rng.standard_normal((L, n)) / 50)
    code = oracle.adaln_code(e, basis)
    mod = oracle.adaln_modulation(code, proj, bias)
    E = _vals_bf16(e)
    B = [[Fraction(float(v)) for v in row] for row in _vals_f16(basis)]
    P = _vals_f16(proj)
    C = _vals_f16(bias)
    for b in range(bt):
        z = [sum(B[j][k] * E[b][k] for k in range(d)) for j in range(r)]
        for j in range(r):
            assert abs(Fraction(float(code[b, j])) - z[j]) <= Fraction(1, 10 ** 14) * (1 + abs(z[j]))
        for l in range(L):
            for i in range(n):
                want = sum(Fraction(float(P[l, i, j])) * z[j] for j in range(r)) + Fraction(float(C[l, i]))
                assert abs(Fraction(float(mod[l, b, i])) - want) <= Fraction(1, 10 ** 14) * (1 + abs(want))


def test_one_hot_and_zero_embeddings():
    """e = unit vector k0 selects column k0 of the basis exactly; e = 0 gives the bias."""
    _, basis, proj, bias = S.adaln_inputs(3, 7, 64, 16, ())
    e = np.zeros((2, 64))
    e[0, 17] = 1.0
    code = oracle.adaln_code(_bf16(e), basis)
    assert np.array_equal(code[0], _vals_f16(basis)[:, 17])
    assert (code[1] == 0).all()
    mod = oracle.adaln_modulation(code, proj, bias)
    assert np.array_equal(mod[:, 1, :], _vals_f16(bias))
    # Without a bias the zero embedding gives exact zeros.
    assert (oracle.adaln_modulation(code, proj, None)[:, 1, :] == 0).all()


def test_integer_data_is_exact():
    """Small integers everywhere: every sum is an exact integer, so the oracle equals
    plain integer arithmetic."""
    rng = np.random.default_rng(12)
    L, n, d, r, bt = 2, 9, 40, 16, 3
    ei = rng.integers(-4, 5, (bt, d))
    bi = rng.integers(-3, 4, (r, d))
    pi = rng.integers(-5, 6, (L, n, r))
    ci = rng.integers(-7, 8, (L, n))
    mod = oracle.adaln_modulation(oracle.adaln_code(_bf16(ei), _f16(bi)), _f16(pi), _f16(ci))
    z = ei.astype(object) @ bi.T.astype(object)
    for l in range(L):
        want = z @ pi[l].T.astype(object) + ci[l].astype(object)[None, :]
        assert np.array_equal(mod[l], want.astype(np.float64))


def test_factorization_equals_dense_projection():
    """The factorized map equals the dense per-block projection W_l = proj_l . basis
    (n x d) that it replaces, applied directly to the embedding."""
    e, basis, proj, bias = S.adaln_inputs(2, 33, 96, 16, S.SAMPLER_TIMESTEPS[:3])
    mod = oracle.adaln_modulation(oracle.adaln_code(e, basis), proj, bias)
    ev = S.bf16_to_f32(e).astype(np.float64)
    for l in range(2):
        W = _vals_f16(proj)[l] @ _vals_f16(basis)          # [n, d]
        dense = ev @ W.T + _vals_f16(bias)[l][None, :]
        np.testing.assert_allclose(mod[l], dense, rtol=1e-12, atol=1e-14)


def test_tolerance_covers_fp32_sequential_sums():
    """A plain FP32 evaluation (one rounding per multiply-add, in index order) stays
    inside the stated bound.  (The bound is worst-case over summation orders and
    scales with sum |basis e|, which cancellation makes ~40x larger than |code| here;
    the GPU tests therefore also use integer data, where every order is exact.)"""
    e, basis, proj, bias = S.adaln_inputs(2, 50, 2688, 16, S.SAMPLER_TIMESTEPS[:2])
    ref = oracle.adaln_modulation(oracle.adaln_code(e, basis), proj, bias)
    tol = oracle.adaln_tolerance(e, basis, proj, bias)
    ev = S.bf16_to_f32(e)
    bv = _vals_f16(basis).astype(np.float32)
    code = np.zeros((2, 16), dtype=np.float32)
    for k in range(2688):
        code = (code + ev[:, k:k + 1] * bv[None, :, k]).astype(np.float32)
    pv = _vals_f16(proj).astype(np.float32)
    out = np.repeat(_vals_f16(bias).astype(np.float32)[:, None, :], 2, axis=1)
    for j in range(16):
        out = (out + pv[:, None, :, j] * code[None, :, j:j + 1]).astype(np.float32)
    assert (np.abs(out.astype(np.float64) - ref) <= tol).all()
