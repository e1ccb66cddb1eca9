"""fh_nvfp4_linear_host: the layer on host buffers, pipelined over row chunks.
Its output must be byte-identical to fh_quantize_act + fh_nvfp4_linear on the
same rows (those two are pinned to the oracle elsewhere), for a single chunk,
whole and ragged multi-chunk inputs, back-to-back calls and pageable memory."""
import numpy as np
import pytest
import torch

import synthetic as S
from _gpu_util import fh

pytestmark = pytest.mark.gpu

K, N = 2688, 1344
SG_A, SG_W = 1.0 / 256, 1.0 / 8192


def _weights():
    m = fh()
    w = torch.from_numpy(S.random_bf16(("host", "w"), (N, K), 0.02).view(np.int16)).cuda().view(torch.bfloat16)
    b = torch.from_numpy(S.random_bf16(("host", "b"), (N,), 0.1).view(np.int16)).cuda().view(torch.bfloat16)
    wc, wsc = m.empty_quantized(N, K)
    m.fh_quantize_act(w, SG_W, wc, wsc, None)
    return wc, wsc, b


def _device_reference(x_host, wc, wsc, b):
    m = fh()
    M = x_host.shape[0]
    x = x_host.cuda()
    ac, asc = m.empty_quantized(M, K)
    clip = torch.zeros(1, dtype=torch.int64, device="cuda")
    m.fh_quantize_act(x, SG_A, ac, asc, clip)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    m.fh_nvfp4_linear(ac, asc, SG_A, wc, wsc, SG_W, b, y)
    torch.cuda.synchronize()
    return y.cpu(), int(clip.item())


def _x(M, tag, pinned=True, scale=1.0):
    bits = S.random_bf16(("host", tag, M), (M, K), scale)
    t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
    return t.pin_memory() if pinned else t.clone()


@pytest.mark.parametrize("M,chunk", [(1000, 4096), (4096, 4096), (9000, 4096), (700, 128)])
def test_host_path_byte_identical_to_device_path(M, chunk):
    m = fh()
    wc, wsc, b = _weights()
    x_host = _x(M, "a", scale=3.0)  # some elements clip at SG_A
    y_host = torch.full((M, N), float("nan"), dtype=torch.bfloat16).pin_memory()
    clip = torch.zeros(1, dtype=torch.int64, device="cuda")
    ws = torch.empty(m.fh_nvfp4_linear_host_workspace_bytes(K, N, chunk), dtype=torch.uint8, device="cuda")
    m.fh_nvfp4_linear_host(x_host, SG_A, wc, wsc, SG_W, b, y_host, clip, chunk_rows=chunk, workspace=ws)
    torch.cuda.synchronize()
    m.fh_device_status()
    y_ref, clips_ref = _device_reference(x_host, wc, wsc, b)
    assert torch.equal(y_host.view(torch.int16), y_ref.view(torch.int16))
    assert int(clip.item()) == clips_ref > 0


def test_back_to_back_calls_and_pageable_memory():
    """Two calls in a row (the slot events are reused) and a call on pageable
    host memory, each checked against the device path."""
    m = fh()
    wc, wsc, b = _weights()
    outs = []
    for tag, pinned in (("b1", True), ("b2", True), ("b3", False)):
        x_host = _x(5000, tag, pinned)
        y_host = torch.empty((5000, N), dtype=torch.bfloat16)
        y_host = y_host.pin_memory() if pinned else y_host
        m.fh_nvfp4_linear_host(x_host, SG_A, wc, wsc, SG_W, b, y_host, None, chunk_rows=1024)
        outs.append((x_host, y_host))
    torch.cuda.synchronize()
    m.fh_device_status()
    for x_host, y_host in outs:
        y_ref, _ = _device_reference(x_host, wc, wsc, b)
        assert torch.equal(y_host.view(torch.int16), y_ref.view(torch.int16))


def test_explicit_stream_with_owned_workspace():
    """A call on a stream other than the current one, with the workspace left
    to the binding: the workspace must stay reserved for that stream's work, so
    allocations made on the current stream right after the call (which would
    reuse a freed block) do not disturb the result."""
    m = fh()
    wc, wsc, b = _weights()
    x_host = _x(9000, "side")
    y_host = torch.empty((9000, N), dtype=torch.bfloat16).pin_memory()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    m.fh_nvfp4_linear_host(x_host, SG_A, wc, wsc, SG_W, b, y_host, None, chunk_rows=1024, stream=side)
    junk = [torch.full((1 << 22,), 7, dtype=torch.int32, device="cuda") for _ in range(8)]
    torch.cuda.synchronize()
    m.fh_device_status()
    del junk
    y_ref, _ = _device_reference(x_host, wc, wsc, b)
    assert torch.equal(y_host.view(torch.int16), y_ref.view(torch.int16))
