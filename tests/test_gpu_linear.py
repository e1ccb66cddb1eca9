"""GPU parity of the tcgen05 NVFP4 linear layer against the oracle's binary64
dequantized product: |y - y_ref| <= 2^-8 |y_ref| + 1e-5 sum_k |a_k w_k| per
output (the oracle quantizes the same BF16 inputs itself; the quantizer's
bit-exactness is checked on the same inputs first)."""
import numpy as np
import pytest
import torch

import oracle
import synthetic as S
from _gpu_util import (bits_of, check_linear, check_quantize, check_quantized, fh, quantize_tiled, sample_rows,
                       tile_rows, to_dev)

pytestmark = pytest.mark.gpu


def run_layer(x_bits, w_bits, b_bits, sg_a, sg_w, keep=None):
    """Quantize x and W on the GPU and run the GEMM.  keep: a dict that receives
    the GPU's activation codes, scales and clip count for a full comparison."""
    m = fh()
    M, K = x_bits.shape
    N = w_bits.shape[0]
    ac, asc, aclip = quantize_tiled(to_dev(x_bits), sg_a)
    wc, wsc, _ = quantize_tiled(to_dev(w_bits), sg_w)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    y.fill_(float("nan"))
    bias = None if b_bits is None else to_dev(b_bits)
    m.fh_nvfp4_linear(ac, asc, sg_a, wc, wsc, sg_w, bias, y)
    torch.cuda.synchronize()
    if keep is not None:
        keep.update(codes=ac, scales=asc)
    return y, int(aclip.item())


SMALL = [(1, 64, 8), (100, 128, 200), (128, 256, 256), (129, 192, 392), (300, 320, 192),
         (257, 2688, 384), (64, 512, 64), (130, 1024, 136)]


@pytest.mark.parametrize("M,K,N", SMALL)
def test_small_and_ragged_shapes(M, K, N):
    x = S.random_bf16(("lin", M, K, "x"), (M, K), 1.0)
    w = S.random_bf16(("lin", M, K, "w"), (N, K), 0.02)
    b = S.random_bf16(("lin", M, K, "b"), (N,), 0.01)
    sg_a = oracle.scale_from_amax(oracle.amax(x))
    sg_w = oracle.scale_from_amax(oracle.amax(w))
    check_quantize(x, sg_a, 1)
    check_quantize(w, sg_w, 1)
    y, _ = run_layer(x, w, b, sg_a, sg_w)
    check_linear(y, x, sg_a, w, sg_w, b)


def test_no_bias_and_unit_scales():
    M, K, N = 130, 256, 200
    x = S.random_bf16(("lin", "nobias", "x"), (M, K), 2.0)
    w = S.random_bf16(("lin", "nobias", "w"), (N, K), 2.0)
    y, _ = run_layer(x, w, None, 1.0, 1.0)
    check_linear(y, x, 1.0, w, 1.0, None)


def test_tiny_workload():
    layer = S.workloads()["tiny"][0]
    calib = S.activation_batches(layer, 0, layer.n_calib)
    sg_a = oracle.scale_from_amax(oracle.amax(calib))
    x = S.activations(layer)
    w, b = S.weights(layer), S.bias(layer)
    sg_w = oracle.scale_from_amax(oracle.amax(w))
    y, clips = run_layer(x, w, b, sg_a, sg_w)
    assert clips == 0
    check_linear(y, x, sg_a, w, sg_w, b)


def layer_case(name, idx=0, calib_batches=None):
    layer = S.workloads()[name][idx]
    x = S.activations(layer)
    n_cal = layer.n_calib if calib_batches is None else calib_batches
    extra = S.activation_batches(layer, layer.n_eval_batches, n_cal - layer.n_eval_batches) \
        if n_cal > layer.n_eval_batches else None
    amax = max(oracle.amax(x), oracle.amax(extra) if extra is not None else 0.0)
    w, b = S.weights(layer), S.bias(layer)
    return layer, x, w, b, oracle.scale_from_amax(amax), oracle.scale_from_amax(oracle.amax(w))


@pytest.mark.parametrize("name", ["attn_proj", "qkv"])
def test_full_size_layer(name):
    """Configs 2 and 3 at their stated sizes: the activation quantizer's whole
    output (codes, scales, clip count) bit-exact against the oracle, the
    weights' too, and the GEMM within tolerance on one row of every 128-row
    tile (every column) plus the tile and matrix edges."""
    layer, x, w, b, sg_a, sg_w = layer_case(name)
    got = {}
    y, clips = run_layer(x, w, b, sg_a, sg_w, keep=got)
    assert clips == 0
    check_quantized(got["codes"], got["scales"], clips, x, sg_a)
    check_quantize(w, sg_w, 1)
    check_linear(y, x, sg_a, w, sg_w, b, rows=tile_rows(layer.M))
    assert not torch.isnan(y).any()


def test_ffn_pair_with_gelu():
    """Config 4 at its stated size: up-projection 32768 x 2688 -> 10752, GELU on
    BF16, the down layer's calibration over the GELU outputs of the same batches
    (reading R10), its quantizer's whole 32768 x 10752 output bit-exact against
    the oracle, and the down-projection.  Both quantizers clip nothing; both
    GEMMs are checked on one row of every 128-row tile plus the edges.  (The up
    layer's inputs carry one outlier of exactly 137 L in every batch, so its
    amax over the evaluation batches equals the amax over all 1000.)"""
    m = fh()
    up = S.workloads()["ffn"][0]
    down = S.workloads()["ffn"][1]
    _, x, w1, b1, sg_x, sg_w1 = layer_case("ffn", 0, calib_batches=up.n_eval_batches)
    w2, b2 = S.weights(down), S.bias(down)
    sg_w2 = oracle.scale_from_amax(oracle.amax(w2))
    got = {}
    h, clips = run_layer(x, w1, b1, sg_x, sg_w1, keep=got)
    assert clips == 0
    check_quantized(got["codes"], got["scales"], clips, x, sg_x)
    check_linear(h, x, sg_x, w1, sg_w1, b1, rows=tile_rows(up.M, salt=1))
    del got
    g = torch.empty_like(h)
    m.fh_gelu_bf16(h, g)
    del h
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    m.fh_amax(g, amax)                         # the down layer's calibration over the same batches
    torch.cuda.synchronize()
    g_bits = bits_of(g)
    assert amax.item() == oracle.amax(g_bits)
    sg_h = m.fh_scale_from_amax(amax.item())
    assert sg_h == oracle.scale_from_amax(amax.item())
    gc, gsc, gclip = quantize_tiled(g, sg_h)   # the 32768 x 10752 launch that feeds the down GEMM
    wc, wsc, _ = quantize_tiled(to_dev(w2), sg_w2)
    y = torch.full((up.M, down.N), float("nan"), dtype=torch.bfloat16, device="cuda")
    m.fh_nvfp4_linear(gc, gsc, sg_h, wc, wsc, sg_w2, to_dev(b2), y)
    torch.cuda.synchronize()
    assert int(gclip.item()) == 0
    check_quantized(gc, gsc, 0, g_bits, sg_h)
    check_quantize(w2, sg_w2, 1)
    check_linear(y, g_bits, sg_h, w2, sg_w2, b2, rows=tile_rows(up.M, salt=2))
    assert not torch.isnan(y).any()


def test_block_sweep_layers_sampled():
    """Two blocks of the 42-block sweep (all four layer shapes), rows sampled."""
    sweep = S.workloads()["block_sweep"]
    for layer in sweep[0:4] + sweep[-4:]:
        small = S.Layer(layer.name, 4096, layer.K, layer.N, layer.batch, 64,
                        channel_lognormal=layer.channel_lognormal, key=layer.key)
        x = S.activations(small)
        w, b = S.weights(layer), S.bias(layer)
        sg_a = oracle.scale_from_amax(oracle.amax(x))
        sg_w = oracle.scale_from_amax(oracle.amax(w))
        y, clips = run_layer(x, w, b, sg_a, sg_w)
        assert clips == 0
        check_linear(y, x, sg_a, w, sg_w, b, rows=sample_rows(small.M, 16))


def test_back_to_back_calls_reuse_nothing():
    """Two different problems in a row on one stream give the same answers as alone."""
    x1 = S.random_bf16(("b2b", 1), (256, 512), 1.0)
    w1 = S.random_bf16(("b2b", 2), (384, 512), 0.02)
    x2 = S.random_bf16(("b2b", 3), (130, 256), 1.0)
    w2 = S.random_bf16(("b2b", 4), (200, 256), 0.02)
    ya, _ = run_layer(x1, w1, None, 0.01, 0.0001)
    yb, _ = run_layer(x2, w2, None, 0.01, 0.0001)
    ya2, _ = run_layer(x1, w1, None, 0.01, 0.0001)
    assert torch.equal(ya.view(torch.int16), ya2.view(torch.int16))
    check_linear(yb, x2, 0.01, w2, 0.0001, None)
    fh().fh_device_status()


def test_single_cta_form_matches_oracle():
    """The single-CTA kernel form (FH_GEMM_CTAS=1: 128-row tiles, cta_group::1)
    passes the same parity cases as the default CTA-pair form."""
    import os
    import subprocess
    import sys
    env = dict(os.environ, FH_GEMM_CTAS="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", os.path.abspath(__file__),
                        "-k", "small or tiny or no_bias or back_to_back or full_size"],
                       env=env, capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]


def test_192_wide_pair_form_matches_oracle():
    """The 256 x 192-tile CTA-pair form (FH_GEMM_BN=192: two accumulators, four
    epilogue warps) passes the same parity cases as the default 256-wide form."""
    import os
    import subprocess
    import sys
    env = dict(os.environ, FH_GEMM_BN="192")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", os.path.abspath(__file__),
                        "-k", "small or tiny or no_bias or back_to_back or full_size"],
                       env=env, capture_output=True, text=True, timeout=1200)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-2000:]


_FORM_HASH = r"""
import hashlib, sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
import nvfp4_quantized_linear_fh_b200 as fh
import synthetic as S
out = []
for (M, K, N) in [(700, 2688, 8064), (333, 1024, 200), (4100, 10752, 2688)]:
    def dev(b):
        return torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).cuda().view(torch.bfloat16)
    x = dev(S.random_bf16(("forms", M, "x"), (M, K), 1.0))
    w = dev(S.random_bf16(("forms", M, "w"), (N, K), 0.02))
    b = dev(S.random_bf16(("forms", M, "b"), (N,), 0.1))
    ac, asc = fh.empty_quantized(M, K); wc, wsc = fh.empty_quantized(N, K)
    fh.fh_quantize_act(x, 1.0 / 256, ac, asc, None); fh.fh_quantize_act(w, 1.0 / 8192, wc, wsc, None)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    fh.fh_nvfp4_linear(ac, asc, 1.0 / 256, wc, wsc, 1.0 / 8192, b, y)
    g, gs = fh.empty_quantized(M, N) if N % 64 == 0 else (None, None)
    if g is not None:
        fh.fh_nvfp4_linear_gelu_quant(ac, asc, 1.0 / 256, wc, wsc, 1.0 / 8192, b, 1.0 / 512, g, gs, None)
    torch.cuda.synchronize()
    h = hashlib.sha256(y.view(torch.int16).cpu().numpy().tobytes())
    if g is not None:
        h.update(g.cpu().numpy().tobytes()); h.update(gs.cpu().numpy().tobytes())
    out.append(h.hexdigest()[:16])
fh.fh_device_status()
print(" ".join(out))
"""


def test_kernel_forms_are_bit_identical():
    """The 256-wide pair form (default), the 192-wide pair form and the
    single-CTA form accumulate in the same order: y, and the fused epilogue's
    codes and scales, are byte-identical across them (ragged M, N and K)."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    hashes = {}
    for name, extra in (("256 pair", {}), ("192 pair", {"FH_GEMM_BN": "192"}), ("single CTA", {"FH_GEMM_CTAS": "1"})):
        env = dict(os.environ, **extra)
        r = subprocess.run([sys.executable, "-c", _FORM_HASH, root], env=env, capture_output=True, text=True,
                           timeout=600)
        assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
        hashes[name] = r.stdout.strip().splitlines()[-1]
    assert len(set(hashes.values())) == 1, hashes


def test_bounded_wait_reports_timeout_and_context_survives():
    """A wait that nothing satisfies gives up after its limit, the host reads
    FH_ERR_TIMEOUT, and the next GEMM still runs correctly."""
    m = fh()
    m.fh_device_status()                      # clean start
    m.fh_selftest_bounded_wait(200000)        # 0.2 s
    with pytest.raises(m.FHError) as e:
        m.fh_device_status()
    assert e.value.status == m.FH_ERR_TIMEOUT
    m.fh_device_status()                      # the word was cleared
    x = S.random_bf16(("timeout", "x"), (130, 256), 1.0)
    w = S.random_bf16(("timeout", "w"), (200, 256), 0.02)
    y, _ = run_layer(x, w, None, 0.01, 0.0001)
    check_linear(y, x, 0.01, w, 0.0001, None)
    m.fh_device_status()


@pytest.mark.parametrize("mode", ["1", "2"])
def test_gemm_stall_times_out_drains_and_context_survives(monkeypatch, mode):
    """Test hook FH_GEMM_TEST_STALL=1: the first CTA pair's MMA warp stops
    issuing after three stages of its first tile, without committing; that
    pair's producers and epilogues run into their bounded waits (about 4 s)
    with copies and MMAs in flight.  FH_GEMM_TEST_STALL=2: the pair's second
    CTA stops loading after two stages, so its producer and the leader's end at
    different stages and the leader must account for the stages only it
    issued.  Either way the kernel drains what it issued and frees TMEM, and
    the host reads FH_ERR_TIMEOUT; with the hook off, the next GEMM in the same
    context passes parity."""
    m = fh()
    m.fh_device_status()                      # clean start
    x = S.random_bf16(("stall", "x"), (1024, 2688), 1.0)
    w = S.random_bf16(("stall", "w"), (1344, 2688), 0.02)
    sg_a = oracle.scale_from_amax(oracle.amax(x))
    sg_w = oracle.scale_from_amax(oracle.amax(w))
    monkeypatch.setenv("FH_GEMM_TEST_STALL", mode)
    run_layer(x, w, None, sg_a, sg_w)
    monkeypatch.delenv("FH_GEMM_TEST_STALL")
    with pytest.raises(m.FHError) as e:
        m.fh_device_status()
    assert e.value.status == m.FH_ERR_TIMEOUT
    y, _ = run_layer(x, w, None, sg_a, sg_w)
    rows = sample_rows(1024, 64, seed=5)
    check_linear(y, x, sg_a, w, sg_w, None, rows=rows)
    m.fh_device_status()


def test_mma_rate_probe_runs_and_stays_below_the_clock_table_peak():
    """The FP4 tensor-rate probe (a measurement aid) runs with and without the
    scale copies, leaves no error behind, and its rate stays below what the
    clock table allows (148 SMs x 16384 FP4 MACs per cycle at 1965 MHz)."""
    m = fh()
    m.fh_device_status()
    for copies in (False, True):
        m.fh_selftest_mma_rate(1000, copies)                  # warm-up
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        pairs = m.fh_selftest_mma_rate(20000, copies)
        e1.record()
        torch.cuda.synchronize()
        m.fh_device_status()
        assert 1 <= pairs <= torch.cuda.get_device_properties(0).multi_processor_count // 2
        rate = pairs * 20000 * 2.0 * 256 * 256 * 256 / (e0.elapsed_time(e1) * 1e-3)
        assert 1e15 < rate < 148 * 16384 * 2 * 1.965e9 * 1.02, rate
