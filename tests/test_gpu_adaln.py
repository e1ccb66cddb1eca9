"""GPU parity of fh_adaln_modulation, the AdaLN timestep conditioning through a
shared low-rank basis (FastH3 Trim, comfyui-wiki news, "What Trim changes": a
shared 2,688 -> 16 basis plus a small per-block projection, stored in FP16).

Random data is compared with the oracle within the worst-case FP32 bound;
integer data, where every summation order is exact, must match exactly, which
catches a dropped or repeated term that the worst-case bound could hide."""
import numpy as np
import pytest
import torch

import oracle
import synthetic as S
from _gpu_util import fh

pytestmark = pytest.mark.gpu


def _dev16(bits, dtype):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(dtype)


def _run(e, basis, proj, bias, guard=64):
    m = fh()
    bt, d = e.shape
    r = basis.shape[0]
    L, n = proj.shape[0], proj.shape[1]
    code = torch.full((bt, r), float("nan"), dtype=torch.float32, device="cuda")
    total = L * bt * n
    buf = torch.full((total + guard,), float("nan"), dtype=torch.float32, device="cuda")
    buf[total:] = 4321.0
    mod = buf[:total].view(L, bt, n)
    m.fh_adaln_modulation(_dev16(e, torch.bfloat16), _dev16(basis, torch.float16), _dev16(proj, torch.float16),
                          None if bias is None else _dev16(bias, torch.float16), code, mod)
    torch.cuda.synchronize()
    m.fh_device_status()
    assert (buf[total:] == 4321.0).all(), "wrote past the end of mod"
    return code.cpu().numpy(), mod.cpu().numpy()


def _check(e, basis, proj, bias):
    code, mod = _run(e, basis, proj, bias)
    ref_code = oracle.adaln_code(e, basis)
    ev = np.abs(S.bf16_to_f32(e).astype(np.float64))
    code_tol = 2688 * 2.0 ** -24 * 1.01 * (ev @ np.abs(oracle.f16_to_f64(basis)).T) + 1e-37
    assert (np.abs(code - ref_code) <= code_tol).all(), "code out of bound"
    ref = oracle.adaln_modulation(ref_code, proj, bias)
    tol = oracle.adaln_tolerance(e, basis, proj, bias)
    err = np.abs(mod.astype(np.float64) - ref)
    bad = np.argwhere(~(err <= tol))
    assert bad.size == 0, f"{len(bad)} modulations out of bound, first at {bad[:3].tolist()}"
    return mod, ref


@pytest.mark.parametrize("L,n,d,r,bt", [(1, 1, 8, 16, 3), (3, 100, 64, 8, 1), (2, 257, 136, 24, 5),
                                        (5, 999, 2688, 32, 130), (4, 16128, 2688, 16, 2)])
def test_matches_oracle(L, n, d, r, bt):
    ts = [int(t) for t in range(bt)]
    e, basis, proj, bias = S.adaln_inputs(L, n, d, r, ts, seed=L + n)
    _check(e, basis, proj, bias)


def test_full_workload_42_blocks_eight_timesteps():
    """42 blocks x 6 x 2688 modulations from the eight sampler timesteps (the launch
    the benchmark times)."""
    e, basis, proj, bias = S.adaln_inputs(42, 6 * 2688, 2688, 16, S.SAMPLER_TIMESTEPS)
    mod, ref = _check(e, basis, proj, bias)
    # Typical FP32 error is far inside the worst-case bound.
    rel = np.abs(mod - ref) / (np.abs(ref) + 1e-3)
    assert np.median(rel) < 1e-5


def test_integer_data_exact():
    rng = np.random.default_rng(21)
    L, n, d, r, bt = 3, 700, 2688, 16, 9
    ei = rng.integers(-4, 5, (bt, d)).astype(np.float64)
    bi = rng.integers(-3, 4, (r, d)).astype(np.float64)
    pi = rng.integers(-5, 6, (L, n, r)).astype(np.float64)
    ci = rng.integers(-7, 8, (L, n)).astype(np.float64)
    e, basis, proj, bias = S.to_bf16_bits(ei), S.to_f16_bits(bi), S.to_f16_bits(pi), S.to_f16_bits(ci)
    code, mod = _run(e, basis, proj, bias)
    ref_code = oracle.adaln_code(e, basis)
    assert np.array_equal(code.astype(np.float64), ref_code)
    assert np.array_equal(mod.astype(np.float64), oracle.adaln_modulation(ref_code, proj, bias))


def test_without_bias():
    e, basis, proj, _ = S.adaln_inputs(2, 300, 256, 16, (999, 125), seed=3)
    _check(e, basis, proj, None)


def test_codes_only():
    """blocks = 0: only the shared code is computed."""
    m = fh()
    e, basis, _, _ = S.adaln_inputs(1, 8, 2688, 16, S.SAMPLER_TIMESTEPS, seed=4)
    code = torch.full((8, 16), float("nan"), dtype=torch.float32, device="cuda")
    proj = torch.empty((0, 8, 16), dtype=torch.float16, device="cuda")
    mod = torch.empty((0, 8, 8), dtype=torch.float32, device="cuda")
    m.fh_adaln_modulation(_dev16(e, torch.bfloat16), _dev16(basis, torch.float16), proj, None, code, mod)
    torch.cuda.synchronize()
    ref = oracle.adaln_code(e, basis)
    ev = np.abs(S.bf16_to_f32(e).astype(np.float64))
    tol = 2688 * 2.0 ** -24 * 1.01 * (ev @ np.abs(oracle.f16_to_f64(basis)).T)
    assert (np.abs(code.cpu().numpy() - ref) <= tol).all()
