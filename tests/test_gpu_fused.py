"""GPU parity of fh_nvfp4_linear_gelu_quant (the NVFP4 linear layer whose
epilogue applies GELU and quantizes the result for the next layer).

Its contract is bit-identity with the three separate calls it replaces,
fh_nvfp4_linear -> fh_gelu_bf16 -> fh_quantize_act, each of which the other GPU
test files pin to the oracle; on small cases the fused codes and scales are also
compared with the oracle's quantization of the same GELU output directly."""
import numpy as np
import pytest
import torch

import oracle
import synthetic as S
from _gpu_util import fh, quantize_tiled, to_dev

pytestmark = pytest.mark.gpu


def _inputs(tag, M, K, N):
    x = S.random_bf16(("fused", tag, "x"), (M, K), 1.0)
    w = S.random_bf16(("fused", tag, "w"), (N, K), 0.03)
    b = S.random_bf16(("fused", tag, "b"), (N,), 0.05)
    return x, w, b


def _run_both(x, w, b, out_scale_factor=1.0):
    """The fused call and the three-call chain on the same quantized operands."""
    m = fh()
    M, K = x.shape
    N = w.shape[0]
    sg_a = oracle.scale_from_amax(oracle.amax(x))
    sg_w = oracle.scale_from_amax(oracle.amax(w))
    ac, asc, _ = quantize_tiled(to_dev(x), sg_a)
    wc, wsc, _ = quantize_tiled(to_dev(w), sg_w)
    bias = to_dev(b)
    # Chain: y, g = GELU(y), then quantize g with the next layer's scale.
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    m.fh_nvfp4_linear(ac, asc, sg_a, wc, wsc, sg_w, bias, y)
    g = torch.empty_like(y)
    m.fh_gelu_bf16(y, g)
    torch.cuda.synchronize()
    g_bits = g.view(torch.int16).cpu().numpy().view(np.uint16)
    # Next layer's global scale: calibrated on g itself, optionally scaled down
    # so that some elements clip.
    sg_o = oracle.scale_from_amax(oracle.amax(g_bits) * out_scale_factor)
    rc, rsc, rclip = quantize_tiled(g, sg_o)
    # Fused, into poisoned buffers.
    oc, osc = m.empty_quantized(M, N)
    oc.fill_(0xA5)
    osc.fill_(0xA5)
    oclip = torch.zeros(1, dtype=torch.int64, device="cuda")
    m.fh_nvfp4_linear_gelu_quant(ac, asc, sg_a, wc, wsc, sg_w, bias, sg_o, oc, osc, oclip)
    torch.cuda.synchronize()
    m.fh_device_status()
    return dict(g_bits=g_bits, sg_o=sg_o, ref=(rc, rsc, int(rclip.item())), got=(oc, osc, int(oclip.item())))


def _assert_identical(r):
    (rc, rsc, rclip), (oc, osc, oclip) = r["ref"], r["got"]
    bad = (rc != oc).nonzero()
    assert bad.numel() == 0, f"{bad.shape[0]} code bytes differ, first {bad[:4].tolist()}"
    bad = (rsc != osc).nonzero()
    assert bad.numel() == 0, f"{bad.shape[0]} scale bytes differ (padding included), first {bad[:4].tolist()}"
    assert oclip == rclip


SHAPES = [(100, 256, 192), (129, 512, 384), (300, 2688, 448), (257, 1024, 128), (64, 128, 64), (513, 768, 576)]


@pytest.mark.parametrize("M,K,N", SHAPES)
def test_fused_matches_three_calls(M, K, N):
    x, w, b = _inputs(("s", M, K, N), M, K, N)
    _assert_identical(_run_both(x, w, b))


@pytest.mark.parametrize("factor", [0.5, 0.1])
def test_fused_clip_counts(factor):
    """A next-layer scale below the calibrated one clips; the counts agree."""
    x, w, b = _inputs(("clip", factor), 260, 512, 320)
    r = _run_both(x, w, b, out_scale_factor=factor)
    assert r["ref"][2] > 0
    _assert_identical(r)


def test_fused_codes_against_oracle():
    """The oracle quantizes the same GELU output and gets the fused codes,
    scales (padding rows zero) and clip count."""
    x, w, b = _inputs("oracle", 150, 512, 256)
    r = _run_both(x, w, b, out_scale_factor=0.5)
    oc_, osc_, oclip_ = oracle.quantize(r["g_bits"], r["sg_o"])
    oc, osc, oclip = r["got"]
    np.testing.assert_array_equal(oc.cpu().numpy(), oc_)
    M, N = r["g_bits"].shape
    gs = osc.cpu().numpy()
    off = oracle.tiled_scale_offsets(M, N)
    np.testing.assert_array_equal(gs[off], osc_)
    rest = np.ones(gs.size, dtype=bool)
    rest[off.reshape(-1)] = False
    assert (gs[rest] == 0).all(), "padding scales must be zero"
    assert oclip == oclip_


def test_fused_ffn_up_full_size():
    """The FFN up projection of the 2688-wide block, 32768 x 2688 -> 10752:
    bit-identical to the three calls on every output byte."""
    layer = S.workloads()["ffn"][0]
    assert (layer.K, layer.N) == (2688, 10752)
    M = 32768
    x = S.random_bf16(("fused", "ffn", "x"), (M, layer.K), 1.0)
    w = S.weights(layer)
    b = S.bias(layer)
    _assert_identical(_run_both(x, w, b))


def test_fused_rejects_bad_shapes():
    m = fh()
    ac, asc = m.empty_quantized(128, 256)
    wc, wsc = m.empty_quantized(200, 256)
    oc, osc = m.empty_quantized(128, 200)
    with pytest.raises(m.FHError) as e:
        m.fh_nvfp4_linear_gelu_quant(ac, asc, 1.0, wc, wsc, 1.0, None, 1.0, oc, osc)
    assert e.value.status == m.FH_ERR_UNSUPPORTED_SHAPE


def test_fused_single_cta_form():
    """The single-CTA kernel form (FH_GEMM_CTAS=1) with the fused epilogue."""
    import os
    import subprocess
    import sys
    env = dict(os.environ, FH_GEMM_CTAS="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", os.path.abspath(__file__),
                        "-k", "matches_three_calls or clip_counts"],
                       env=env, capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]


def test_fused_192_wide_pair_form():
    """The 256 x 192-tile CTA-pair form (FH_GEMM_BN=192) with the fused epilogue."""
    import os
    import subprocess
    import sys
    env = dict(os.environ, FH_GEMM_BN="192")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", os.path.abspath(__file__),
                        "-k", "matches_three_calls or clip_counts"],
                       env=env, capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]


# The last two shapes give the quantizer's CTAs 4 wide (128-column) and 13 narrow
# (64-column) units each on a 148-SM B200, with ragged row blocks.
@pytest.mark.parametrize("M,K", [(100, 192), (129, 512), (300, 2688), (1, 64), (513, 10752), (5757, 2688), (11483, 2624)])
def test_gelu_quantize_matches_two_calls(M, K):
    """fh_gelu_quantize_act == fh_gelu_bf16 then fh_quantize_act, bit for bit
    (codes, every scale byte including padding rows, clip count)."""
    m = fh()
    y = to_dev(S.random_bf16(("gq", M, K), (M, K), 2.0))
    g = torch.empty_like(y)
    m.fh_gelu_bf16(y, g)
    torch.cuda.synchronize()
    g_bits = g.view(torch.int16).cpu().numpy().view(np.uint16)
    sg = oracle.scale_from_amax(oracle.amax(g_bits) * 0.5)
    rc, rsc, rclip = quantize_tiled(g, sg)
    oc, osc = m.empty_quantized(M, K)
    oc.fill_(0xA5)
    osc.fill_(0xA5)
    oclip = torch.zeros(1, dtype=torch.int64, device="cuda")
    m.fh_gelu_quantize_act(y, sg, oc, osc, oclip)
    torch.cuda.synchronize()
    m.fh_device_status()
    _assert_identical(dict(ref=(rc, rsc, int(rclip.item())), got=(oc, osc, int(oclip.item()))))
    if M * K <= 300 * 2688:  # and the oracle's quantization of the same GELU output
        oc_, osc_, oclip_ = oracle.quantize(g_bits, sg)
        np.testing.assert_array_equal(oc.cpu().numpy(), oc_)
        assert int(oclip.item()) == oclip_
