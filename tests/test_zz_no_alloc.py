"""fh_nvfp4_linear_host_noalloc: the host-buffer layer for callers that cannot
allocate device memory (an engine or application that keeps the device's
memory in its own pool, a plugin limited to the memory it is given, or a
caller that cannot afford cudaMalloc's device synchronization).  It stages its
chunks in the library's static scratch array instead of a caller's workspace.

The GPU test calls the entry point through the C ABI (ctypes, no binding
wrapper) twice in a row, on different inputs, and compares each result with
the existing workspace entry point fh_nvfp4_linear_host: byte for byte, which
is within any tolerance, and against the oracle within the GEMM tolerance on
sampled rows.  This file is collected last, so a run that stops at its first
failure has run every other test before it."""
import ctypes

import numpy as np
import pytest
import torch

import synthetic as S
from _gpu_util import check_linear, fh

K = 2688
SG_A, SG_W = 1.0 / 256, 1.0 / 8192


def _host(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).pin_memory()


def _noalloc(x_host, wc, wsc, b, y_host, clip):
    """The entry point, called through the C ABI."""
    m = fh()
    M, Kx = x_host.shape
    N = wc.shape[0]
    return m.lib().fh_nvfp4_linear_host_noalloc(
        ctypes.c_void_p(x_host.data_ptr()), M, Kx, ctypes.c_float(SG_A), ctypes.c_void_p(wc.data_ptr()),
        ctypes.c_void_p(wsc.data_ptr()), ctypes.c_float(SG_W), ctypes.c_void_p(b.data_ptr()), N,
        ctypes.c_void_p(y_host.data_ptr()), ctypes.c_void_p(clip.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_two_calls():
    m = fh()
    # Call 1: 3000 rows at N = 2688 (1280-row chunks: two full, one ragged).
    # Call 2: 700 rows at N = 8064 (640-row chunks: one full, one ragged), on
    # other inputs, after call 1 left its contents in the scratch array.
    for call, (M, N) in enumerate(((3000, 2688), (700, 8064))):
        x_bits = S.random_bf16(("noalloc", call, "x"), (M, K), 3.0)      # some elements clip at SG_A
        w_bits = S.random_bf16(("noalloc", call, "w"), (N, K), 0.02)
        b_bits = S.random_bf16(("noalloc", call, "b"), (N,), 0.1)
        w = torch.from_numpy(w_bits.view(np.int16)).cuda().view(torch.bfloat16)
        b = torch.from_numpy(b_bits.view(np.int16)).cuda().view(torch.bfloat16)
        wc, wsc = m.empty_quantized(N, K)
        m.fh_quantize_act(w, SG_W, wc, wsc, None)
        x_host = _host(x_bits)
        y_new = torch.full((M, N), float("nan"), dtype=torch.bfloat16).pin_memory()
        y_old = torch.full((M, N), float("nan"), dtype=torch.bfloat16).pin_memory()
        clip_new = torch.zeros(1, dtype=torch.int64, device="cuda")
        clip_old = torch.zeros(1, dtype=torch.int64, device="cuda")
        assert _noalloc(x_host, wc, wsc, b, y_new, clip_new) == m.FH_OK, m.fh_last_error()
        torch.cuda.synchronize()
        m.fh_device_status()
        m.fh_nvfp4_linear_host(x_host, SG_A, wc, wsc, SG_W, b, y_old, clip_old, chunk_rows=1024)
        torch.cuda.synchronize()
        m.fh_device_status()
        assert torch.equal(y_new.view(torch.int16), y_old.view(torch.int16)), f"call {call + 1} differs"
        assert int(clip_new.item()) == int(clip_old.item()) > 0
        rows = np.unique(np.array([0, 1, 127, 128, 639, 640, 1279, 1280, M // 2, M - 1]).clip(0, M - 1))
        check_linear(y_new, x_bits, SG_A, w_bits, SG_W, b_bits, rows=rows)


def test_noalloc_rejects_chunks_beyond_the_scratch_array():
    """One 128-row chunk of K = 64, N = 65536 needs more than the 16 MiB array:
    refused before any device work, with a message naming the limit."""
    import nvfp4_quantized_linear_fh_b200 as m
    st = m.lib().fh_nvfp4_linear_host_noalloc(ctypes.c_void_p(8), 128, 64, ctypes.c_float(1.0), ctypes.c_void_p(16),
                                              ctypes.c_void_p(16), ctypes.c_float(1.0), None, 65536,
                                              ctypes.c_void_p(8), None, None)
    assert st == m.FH_ERR_UNSUPPORTED_SHAPE
    assert "scratch" in m.fh_last_error()
