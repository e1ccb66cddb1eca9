"""fh_nvfp4_linear_fused_quant: the quantization of the BF16 input fused into
the GEMM kernel.  Its outputs -- y, the activation codes and scales, the clip
count -- must be byte-identical to fh_quantize_act followed by fh_nvfp4_linear
(both pinned to the oracle elsewhere), and are checked against the oracle
directly as well; the sync scratch must come back zero after every call."""
import numpy as np
import pytest
import torch

import oracle
import synthetic as S
from _gpu_util import check_linear, check_quantized, fh, tile_rows, to_dev

pytestmark = pytest.mark.gpu


def _weights(K, N, tag, sg_w=None):
    m = fh()
    w_bits = S.random_bf16(("fused-pro", tag, "w"), (N, K), 0.02)
    b_bits = S.random_bf16(("fused-pro", tag, "b"), (N,), 0.1)
    sg_w = sg_w or oracle.scale_from_amax(oracle.amax(w_bits))
    wc, wsc = m.empty_quantized(N, K)
    m.fh_quantize_act(to_dev(w_bits), sg_w, wc, wsc, None)
    return w_bits, b_bits, wc, wsc, sg_w


def _both_paths(x, sg_a, wc, wsc, sg_w, b, N, sync=None):
    """(fused y, codes, scales, clips), (separate y, codes, scales, clips) on the same device input."""
    m = fh()
    M, K = x.shape
    sync = m.empty_fused_sync(M) if sync is None else sync
    y1 = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    c1, s1 = m.empty_quantized(M, K)
    s1.fill_(0xA5)
    k1 = torch.zeros(1, dtype=torch.int64, device="cuda")
    m.fh_nvfp4_linear_fused_quant(x, sg_a, wc, wsc, sg_w, b, y1, c1, s1, k1, sync)
    y2 = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    c2, s2 = m.empty_quantized(M, K)
    k2 = torch.zeros(1, dtype=torch.int64, device="cuda")
    m.fh_quantize_act(x, sg_a, c2, s2, k2)
    m.fh_nvfp4_linear(c2, s2, sg_a, wc, wsc, sg_w, b, y2)
    torch.cuda.synchronize()
    m.fh_device_status()
    assert int(sync.abs().sum().item()) == 0, "the sync scratch must be zero after the call"
    return (y1, c1, s1, int(k1.item())), (y2, c2, s2, int(k2.item()))


def _assert_identical(a, b):
    assert torch.equal(a[0].view(torch.int16), b[0].view(torch.int16)), "y differs from the separate calls"
    assert torch.equal(a[1], b[1]), "codes differ from fh_quantize_act"
    assert torch.equal(a[2], b[2]), "scales differ from fh_quantize_act"
    assert a[3] == b[3]


@pytest.mark.parametrize("M,K,N", [(1, 64, 8), (100, 128, 200), (129, 256, 392), (300, 2688, 384),
                                   (1000, 1024, 136), (257, 192, 264), (4100, 2688, 2688)])
def test_matches_separate_calls_and_oracle(M, K, N):
    x_bits = S.random_bf16(("fused-pro", M, K, "x"), (M, K), 3.0)
    sg_a = 1.0 / 256          # some elements clip
    w_bits, b_bits, wc, wsc, sg_w = _weights(K, N, (M, K, N))
    fused, separate = _both_paths(to_dev(x_bits), sg_a, wc, wsc, sg_w, to_dev(b_bits), N)
    _assert_identical(fused, separate)
    check_quantized(fused[1], fused[2], fused[3], x_bits, sg_a)
    rows = tile_rows(M) if M > 256 else np.arange(M)
    check_linear(fused[0], x_bits, sg_a, w_bits, sg_w, b_bits, rows=rows)


def test_strided_input_and_sync_reuse():
    """x inside wider rows (ldx > K); three calls in a row share one sync buffer."""
    m = fh()
    M, K, N = 700, 512, 264
    w_bits, b_bits, wc, wsc, sg_w = _weights(K, N, "strided")
    sync = m.empty_fused_sync(M)
    for i in range(3):
        x_bits = S.random_bf16(("fused-pro", "strided", i), (M, K), 1.0)
        x = to_dev(x_bits, ldx=K + 64)
        assert x.stride(0) == K + 64
        fused, separate = _both_paths(x, 0.002, wc, wsc, sg_w, to_dev(b_bits), N, sync=sync)
        _assert_identical(fused, separate)


def test_qkv_workload_full_size():
    """The fused-QKV workload at its stated size (32768 x 2688 -> 8064), calibrated."""
    m = fh()
    layer = S.workloads()["qkv"][0]
    x = S.activation_batches_t(layer, 0, layer.n_eval_batches, "cuda").view(torch.bfloat16)
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    m.fh_amax(x, amax)
    sg_a = m.fh_scale_from_amax(amax.item())
    w = S.weights_t(layer, "cuda").view(torch.bfloat16)
    wamax = torch.zeros(1, dtype=torch.float32, device="cuda")
    m.fh_amax(w, wamax)
    sg_w = m.fh_scale_from_amax(wamax.item())
    wc, wsc = m.empty_quantized(layer.N, layer.K)
    m.fh_quantize_act(w, sg_w, wc, wsc, None)
    b = S.bias_t(layer, "cuda").view(torch.bfloat16)
    fused, separate = _both_paths(x, sg_a, wc, wsc, sg_w, b, layer.N)
    _assert_identical(fused, separate)
    assert fused[3] == 0
    x_bits = x.view(torch.int16).cpu().numpy().view(np.uint16)
    w_bits = w.view(torch.int16).cpu().numpy().view(np.uint16)
    b_bits = b.view(torch.int16).cpu().numpy().view(np.uint16)
    check_linear(fused[0], x_bits, sg_a, w_bits, sg_w, b_bits, rows=tile_rows(layer.M, salt=7))
