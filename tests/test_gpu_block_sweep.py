"""Config 5 at its stated size: the 42-block sweep, 168 NVFP4 linear layers
(QKV 2688 -> 8064, out-projection 2688 -> 2688, FFN up 2688 -> 10752, FFN down
10752 -> 2688 per block) run back to back at M = 49152 tokens, each layer with
its own seeded weights, its own calibrated activation scale (amax over its
1000-batch calibration stream, whose first 768 batches are the layer's input)
and its input quantized from BF16 (FastH3 Trim, "What Trim changes": 42 blocks;
FastH3 thread digest, tweet 6/8: calibrated scales clip nothing).

Inputs are drawn on the GPU with the torch restatement of the seeded recipes;
the oracle always receives the very BF16 bytes the GPU consumed.  Checks:
  - every layer: the activation clip count is 0 and equals the oracle's count
    on the layer's input; the global scales follow from the amaxes by the
    oracle's rule; the input's oracle amax does not exceed the calibrated one;
    the GEMM output is within tolerance on 24 rows spread over the tiles;
  - blocks 0 and 41 (all four layer shapes): the calibrated amax equals the
    oracle's amax over the whole calibration stream, the activation and weight
    quantizations are bit-exact on every element, and the GEMM is checked on
    one row of every 128-row tile plus the edges (every column)."""
import numpy as np
import pytest
import torch

import oracle
import synthetic as S
from _gpu_util import bits_of, check_linear, check_quantized, fh, tile_rows

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

FULL_BLOCKS = (0, 41)


def spread_rows(M: int, layer_index: int, n: int = 24) -> np.ndarray:
    """n rows in n different 128-row tiles; the tiles move with the layer, so
    over the sweep every tile of every layer shape is visited."""
    tiles = (layer_index * 131 + np.arange(n) * ((M // 128) // n)) % (M // 128)
    return np.unique(tiles * 128 + (layer_index * 7 + np.arange(n) * 29) % 128).astype(np.int64)


def test_block_sweep_full_size():
    m = fh()
    dev = torch.device("cuda")
    sweep = S.workloads()["block_sweep"]
    assert len(sweep) == 168
    for li, layer in enumerate(sweep):
        blk = li // 4
        M, K, N = layer.M, layer.K, layer.N
        full = blk in FULL_BLOCKS
        # Weights and bias (offline): the weight scale from W's own amax.
        w = S.weights_t(layer, dev).view(torch.bfloat16)
        b = S.bias_t(layer, dev).view(torch.bfloat16)
        wamax = torch.zeros(1, dtype=torch.float32, device=dev)
        m.fh_amax(w, wamax)
        sg_w = m.fh_scale_from_amax(wamax.item())
        wc, wsc = m.empty_quantized(N, K)
        wclip = torch.zeros(1, dtype=torch.int64, device=dev)
        m.fh_quantize_act(w, sg_w, wc, wsc, wclip)
        # Calibration: amax over the layer's 1000 batches; the first 768 are its input.
        x = S.activation_batches_t(layer, 0, layer.n_eval_batches, dev).view(torch.bfloat16)
        amax = torch.zeros(1, dtype=torch.float32, device=dev)
        m.fh_amax(x, amax)
        rest_max = 0.0
        for b0 in range(layer.n_eval_batches, layer.n_calib, 116):
            nb = min(116, layer.n_calib - b0)
            xr = S.activation_batches_t(layer, b0, nb, dev).view(torch.bfloat16)
            m.fh_amax(xr, amax)
            if full:
                rest_max = max(rest_max, oracle.amax(bits_of(xr)))
            del xr
        sg_a = m.fh_scale_from_amax(amax.item())
        # The layer: quantize the BF16 input, multiply.
        ac, asc = m.empty_quantized(M, K)
        clip = torch.zeros(1, dtype=torch.int64, device=dev)
        m.fh_quantize_act(x, sg_a, ac, asc, clip)
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=dev)
        m.fh_nvfp4_linear(ac, asc, sg_a, wc, wsc, sg_w, b, y)
        torch.cuda.synchronize()
        # Against the oracle, on the bytes the GPU consumed.
        x_bits, w_bits, b_bits = bits_of(x), bits_of(w), bits_of(b)
        del x, w, b
        gpu_amax = amax.item()
        x_amax = oracle.amax(x_bits)
        assert sg_a == oracle.scale_from_amax(gpu_amax), layer.name
        assert sg_w == oracle.scale_from_amax(oracle.amax(w_bits)), layer.name
        assert x_amax <= gpu_amax, layer.name
        clips = int(clip.item())
        assert clips == oracle.clip_count(x_bits, sg_a) == 0, layer.name
        if full:
            assert gpu_amax == max(x_amax, rest_max), layer.name
            check_quantized(ac, asc, clips, x_bits, sg_a)
            check_quantized(wc, wsc, int(wclip.item()), w_bits, sg_w)
            rows = tile_rows(M, salt=li)
        else:
            rows = spread_rows(M, li)
        check_linear(y, x_bits, sg_a, w_bits, sg_w, b_bits, rows=rows)
        assert not torch.isnan(y).any(), layer.name
        del ac, asc, y, wc, wsc
    m.fh_device_status()
