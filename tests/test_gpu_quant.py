"""GPU parity of the NVFP4 quantizer, the calibration amax, the scale relayout
and the BF16 GELU against the CPU oracle (bit-exact where the output is a code,
a scale or a count)."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import synthetic as S
from _gpu_util import check_quantize, fh, to_dev

pytestmark = pytest.mark.gpu

ROW, TILED = 0, 1


def test_library_is_native():
    m = fh()
    assert m.fh_version() >= 10000
    assert os.path.dirname(m.LIB_PATH) == os.path.dirname(m.__file__)


def golden_rows(pad_to=64):
    """The hand-worked blocks, each padded with zeros to one row of pad_to elements."""
    with open(os.path.join(os.path.dirname(__file__), "golden", "nvfp4_block_cases.json")) as f:
        cases = json.load(f)["cases"]
    return [(c, S.to_bf16_bits(np.array(c["x"] + [0.0] * (pad_to - 16))).reshape(1, -1)) for c in cases]


@pytest.mark.parametrize("layout", [ROW, TILED])
def test_golden_blocks(layout):
    m = fh()
    for c, x in golden_rows():
        check_quantize(x, c["sg"], layout)
        codes, scales = m.empty_quantized(1, 64, layout=layout)
        clip = torch.zeros(1, dtype=torch.int64, device="cuda")
        m.fh_quantize_act(to_dev(x), c["sg"], codes, scales, clip, layout)
        torch.cuda.synchronize()
        assert codes.cpu().numpy()[0, :8].tobytes().hex() == c["codes"], c["name"]
        assert scales.cpu().numpy()[0] == int(c["scale"], 16), c["name"]
        assert clip.item() == c["clip"], c["name"]


SHAPES = [(1, 16), (17, 48), (129, 64), (300, 256), (64, 2688), (200, 448)]


@pytest.mark.parametrize("M,K", SHAPES)
@pytest.mark.parametrize("layout", [ROW, TILED])
def test_random_blocks_assorted_magnitudes(M, K, layout):
    if layout == TILED and K % 64:
        pytest.skip("tensor-core layout needs K % 64 == 0")
    rng = np.random.default_rng(M * 7 + K)
    nb = K // 16
    mags = np.exp(rng.uniform(np.log(1e-5), np.log(3e3), (M, nb, 1)))
    xs = (rng.standard_normal((M, nb, 16)) * mags).reshape(M, K)
    x = S.to_bf16_bits(xs)
    for sg in [float(np.float32(0.0123)), 1.0, 2.0 ** -7, oracle.scale_from_amax(oracle.amax(x))]:
        check_quantize(x, sg, layout)


@pytest.mark.parametrize("layout", [ROW, TILED])
def test_exact_ties_at_many_scales(layout):
    """Every element on an exact E2M1 midpoint at non-power-of-two block scales:
    the converter path cannot decide these and the exact path must."""
    rng = np.random.default_rng(1)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    rows = []
    for sv in [1.125, 1.25, 1.375, 1.5, 1.625, 1.75, 1.875, 0.75, 3.0, 5.0, 13.0, 0.15625, 26.0, 104.0]:
        blocks = []
        for _ in range(4):
            v = rng.choice(mids, 16) * sv * rng.choice([-1.0, 1.0], 16)
            v[rng.integers(16)] = 6 * sv
            blocks.append(v)
        rows.append(np.concatenate(blocks))
    x = S.to_bf16_bits(np.array(rows))
    for sg in [1.0, 0.5, 2.0 ** -10]:
        check_quantize(S.to_bf16_bits(S.bf16_to_f32(x).astype(np.float64) * sg), sg, layout)


def test_row_stride_larger_than_k():
    x = S.random_bf16(("gpu", "ldx"), (33, 128), 2.0)
    check_quantize(x, 0.004, TILED, ldx=200)
    check_quantize(x, 0.004, ROW, ldx=136)


def test_tiny_workload_clip_counts():
    layer = S.workloads()["tiny"][0]
    m = fh()
    calib = S.activation_batches(layer, 0, layer.n_calib)
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    for b in range(layer.n_calib):
        m.fh_amax(to_dev(calib[b * layer.batch:(b + 1) * layer.batch]), amax)
    torch.cuda.synchronize()
    assert amax.item() == oracle.amax(calib)
    sg = m.fh_scale_from_amax(amax.item())
    assert sg == oracle.scale_from_amax(amax.item())
    x = S.activations(layer)
    assert check_quantize(x, sg, TILED) == 0
    pos = S.outlier_positions(layer, 0)
    sg_unc = oracle.scale_from_amax(oracle.amax(np.delete(x.reshape(-1), pos)))
    assert check_quantize(x, sg_unc, TILED) == 33


# The tensor-core-layout quantizer runs 2 CTAs per SM over units of 128 rows x
# 128 columns (3-stage ring) or, when K is an odd multiple of 64, 128 x 64
# (6-stage ring); each unit's scale atoms leave through a staging buffer once
# its ring stage is released.  On a 148-SM B200 these shapes give the CTAs 3,
# 4 and 7 wide units, and 13 or 4 narrow ones: every ring position, the
# end-of-loop stores and ragged row blocks.
@pytest.mark.parametrize("M,K", [(3840, 2688), (5757, 2688), (11259, 2688), (11483, 2624), (2766, 2624)])
def test_tiled_unit_counts(M, K):
    x = S.random_bf16(("tiled-units", M, K), (M, K), 2.0)
    sg = oracle.scale_from_amax(oracle.amax(x))
    assert check_quantize(x, sg, TILED) == 0
    assert check_quantize(x, sg / 64, TILED) > 0


@pytest.mark.parametrize("name", ["attn_proj", "qkv"])
def test_full_size_quantizer(name):
    layer = S.workloads()[name][0]
    x = S.activations(layer)
    calib_amax = oracle.amax(x)
    sg = oracle.scale_from_amax(calib_amax)
    assert check_quantize(x, sg, TILED) == 0


def test_amax_shapes():
    m = fh()
    for shape, ldx in [((1, 1), 1), ((7, 13), 13), ((64, 2688), 2688), ((33, 40), 48)]:
        x = S.random_bf16(("gpu", "amax", shape), shape, 3.0)
        amax = torch.zeros(1, dtype=torch.float32, device="cuda")
        m.fh_amax(to_dev(x, ldx), amax)
        torch.cuda.synchronize()
        assert amax.item() == oracle.amax(x)


def test_scales_to_rowmajor():
    m = fh()
    x = S.random_bf16(("gpu", "relayout"), (300, 320), 1.0)
    codes, scales, _ = __import__("_gpu_util").gpu_quantize(to_dev(x), 0.01, TILED)
    rm = torch.empty(300 * 20, dtype=torch.uint8, device="cuda")
    m.fh_scales_to_rowmajor(scales, rm, 300, 320)
    torch.cuda.synchronize()
    _, osc, _ = oracle.quantize(x, 0.01)
    np.testing.assert_array_equal(rm.cpu().numpy().reshape(300, 20), osc)


def test_gelu_against_oracle():
    m = fh()
    x = S.random_bf16(("gpu", "gelu"), (4096 + 5,), 3.0)
    xd = to_dev(x)
    y = torch.empty_like(xd)
    m.fh_gelu_bf16(xd, y)
    torch.cuda.synchronize()
    ref = oracle.gelu(x)
    got = S.bf16_to_f32(y.view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)
    assert (np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-37).all()


def test_device_status_clean():
    fh().fh_device_status()
