"""The C-ABI library loads without a GPU, exports every entry point that
include/fh.h declares, and its host-only logic (scale rule, buffer sizes,
argument validation) behaves as documented.  No call here reaches a GPU."""
import ctypes
import math
import os
import re

import numpy as np
import pytest

import oracle
import synthetic as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "fh_build", os.path.join(ROOT, "nvfp4_quantized_linear_fh_b200", "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)
    path = build.build()
    L = ctypes.CDLL(path)
    L.fh_scale_from_amax.restype = ctypes.c_float
    L.fh_scale_from_amax.argtypes = [ctypes.c_float]
    L.fh_scales_bytes.restype = ctypes.c_size_t
    L.fh_scales_bytes.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int]
    L.fh_last_error.restype = ctypes.c_char_p
    return L


def declared_entry_points():
    with open(os.path.join(ROOT, "include", "fh.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:int|float|size_t|const char\*)\s+(fh_\w+)\(", text, re.M)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_entry_points()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n


def test_binding_wraps_every_entry_point():
    import nvfp4_quantized_linear_fh_b200 as fh
    for n in declared_entry_points():
        assert callable(getattr(fh, n)), n


def test_scale_from_amax_matches_oracle(lib):
    rng = np.random.default_rng(0)
    vals = np.concatenate([[0.0, 2688.0, 1344.0, 1096.0, 4.5, 1e-30, 3e38],
                           np.exp(rng.uniform(np.log(1e-8), np.log(1e8), 2000))]).astype(np.float32)
    for a in vals:
        assert lib.fh_scale_from_amax(float(a)) == oracle.scale_from_amax(float(a)), a
    assert math.isnan(lib.fh_scale_from_amax(-1.0))
    assert math.isnan(lib.fh_scale_from_amax(float("inf")))


def test_scales_bytes(lib):
    assert lib.fh_scales_bytes(100, 48, 0) == 300
    assert lib.fh_scales_bytes(100, 64, 1) == 128 * 4
    assert lib.fh_scales_bytes(129, 2688, 1) == oracle.tiled_scales_bytes(129, 2688) == 256 * 168
    assert lib.fh_scales_bytes(10, 48, 1) == 0      # K % 64 != 0
    assert lib.fh_scales_bytes(10, 20, 0) == 0      # K % 16 != 0
    assert lib.fh_scales_bytes(10, 64, 7) == 0


def test_argument_validation_without_gpu(lib):
    """Malformed calls are rejected before any device work."""
    P = ctypes.c_void_p
    fake = P(16)
    # fh_quantize_act(x, M, K, ldx, sg, codes, scales, clip, layout, stream)
    q = lib.fh_quantize_act
    q.argtypes = [P, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_float, P, P, P, ctypes.c_int, P]
    assert q(fake, 4, 24, 24, 1.0, fake, fake, None, 0, None) == 2            # K % 16
    assert q(fake, 4, 48, 48, 1.0, fake, fake, None, 1, None) == 2            # tiled needs K % 64
    assert q(fake, 4, 64, 60, 1.0, fake, fake, None, 0, None) == 2            # ldx < K
    assert q(fake, 4, 64, 64, 0.0, fake, fake, None, 0, None) == 1            # scale <= 0
    assert q(fake, 4, 64, 64, float("nan"), fake, fake, None, 0, None) == 1
    assert q(fake, 4, 64, 64, 1.0, fake, fake, None, 5, None) == 1            # layout
    assert q(None, 4, 64, 64, 1.0, fake, fake, None, 0, None) == 1            # null x
    assert q(P(18), 4, 64, 64, 1.0, fake, fake, None, 0, None) == 2          # misaligned
    assert q(fake, 0, 64, 64, 1.0, fake, fake, None, 0, None) == 0            # empty: nothing to do
    assert b"16-byte" in lib.fh_last_error() or lib.fh_last_error() == b""
    g = lib.fh_nvfp4_linear
    g.argtypes = [P, P, ctypes.c_float, P, P, ctypes.c_float, P, P, ctypes.c_int64, ctypes.c_int64,
                  ctypes.c_int64, P]
    assert g(fake, fake, 1.0, fake, fake, 1.0, None, fake, 128, 256, 96, None) == 2   # K % 64
    assert g(fake, fake, 1.0, fake, fake, 1.0, None, fake, 128, 250, 128, None) == 2  # N % 8
    assert g(fake, fake, -1.0, fake, fake, 1.0, None, fake, 128, 256, 128, None) == 1
    assert g(None, fake, 1.0, fake, fake, 1.0, None, fake, 128, 256, 128, None) == 1
    assert g(fake, fake, 1.0, fake, fake, 1.0, None, fake, 0, 256, 128, None) == 0    # empty
    assert g(fake, fake, 1.0, fake, fake, 1.0, None, fake, 128, 0, 128, None) == 0
    f = lib.fh_nvfp4_linear_gelu_quant
    f.argtypes = [P, P, ctypes.c_float, P, P, ctypes.c_float, P, ctypes.c_float, P, P, P,
                  ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, P]
    assert f(fake, fake, 1.0, fake, fake, 1.0, None, 1.0, fake, fake, None, 128, 200, 128, None) == 2  # N % 64
    assert f(fake, fake, 1.0, fake, fake, 1.0, None, 1.0, fake, fake, None, 128, 256, 96, None) == 2   # K % 64
    assert f(fake, fake, 1.0, fake, fake, 1.0, None, 0.0, fake, fake, None, 128, 256, 128, None) == 1  # out scale
    assert f(fake, fake, 1.0, fake, fake, 1.0, None, float("inf"), fake, fake, None, 128, 256, 128, None) == 1
    assert f(fake, fake, 1.0, fake, fake, 1.0, None, 1.0, None, fake, None, 128, 256, 128, None) == 1  # null codes
    assert f(fake, fake, 1.0, fake, fake, 1.0, None, 1.0, P(24), fake, None, 128, 256, 128, None) == 2
    assert f(fake, fake, 1.0, fake, fake, 1.0, None, 1.0, fake, fake, None, 0, 256, 128, None) == 0   # empty
    r = lib.fh_quantize_int8_rows
    r.argtypes = [P, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, P, P, P]
    assert r(fake, 4, 12, 12, fake, fake, None) == 2       # d % 8
    assert r(fake, 4, 16, 8, fake, fake, None) == 2        # ldx < d
    assert r(fake, 4, 16, 20, fake, fake, None) == 2       # ldx % 8
    assert r(None, 4, 16, 16, fake, fake, None) == 1       # null x
    assert r(fake, 4, 16, 16, P(24), fake, None) == 2      # q misaligned
    assert r(fake, 4, 16, 16, fake, P(18), None) == 2      # scales misaligned
    assert r(fake, 0, 16, 16, fake, fake, None) == 0       # empty
    s = lib.fh_int8_attention_scores
    s.argtypes = [P, P, P, P, ctypes.c_float, P, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, P]
    assert s(fake, fake, fake, fake, 1.0, fake, 2, 100, 256, 120, None) == 2   # d % 16
    assert s(fake, fake, fake, fake, 1.0, fake, 2, 100, 256, 131072, None) == 2  # d too large for INT32 sums
    assert s(fake, fake, fake, fake, float("nan"), fake, 2, 100, 256, 128, None) == 1
    assert s(fake, None, fake, fake, 1.0, fake, 2, 100, 256, 128, None) == 1  # null q scales
    assert s(fake, fake, P(40), fake, 1.0, fake, 2, 100, 256, 128, None) == 2  # k misaligned
    assert s(fake, fake, fake, fake, 1.0, fake, 2, 0, 256, 128, None) == 0     # empty
    assert s(fake, fake, fake, fake, 1.0, fake, 0, 100, 256, 128, None) == 0
    d = lib.fh_adaln_modulation
    d.argtypes = [P, ctypes.c_int64, ctypes.c_int64, P, ctypes.c_int64, P, P, ctypes.c_int64, ctypes.c_int64, P, P, P]
    assert d(fake, 8, 2688, fake, 12, fake, None, 42, 16128, fake, fake, None) == 2   # rank not in {8,16,24,32}
    assert d(fake, 8, 2684, fake, 16, fake, None, 42, 16128, fake, fake, None) == 2   # d % 8
    assert d(fake, 8, 2688, fake, 16, fake, None, 1 << 20, 1 << 12, fake, fake, None) == 2  # blocks * n >= 2^31
    assert d(fake, 8, 2688, None, 16, fake, None, 42, 16128, fake, fake, None) == 1   # null basis
    assert d(fake, 8, 2688, fake, 16, P(24), None, 42, 16128, fake, fake, None) == 2  # proj misaligned
    assert d(fake, 8, 2688, fake, 16, fake, P(17), 42, 16128, fake, fake, None) == 2  # bias misaligned
    assert d(fake, 0, 2688, fake, 16, fake, None, 42, 16128, fake, fake, None) == 0   # no timesteps
    hl = lib.fh_nvfp4_linear_host
    hl.argtypes = [P, ctypes.c_int64, ctypes.c_int64, ctypes.c_float, P, P, ctypes.c_float, P, ctypes.c_int64, P, P,
                   ctypes.c_int64, P, ctypes.c_size_t, P]
    wsb = lib.fh_nvfp4_linear_host_workspace_bytes
    wsb.restype = ctypes.c_size_t
    wsb.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64]
    assert wsb(2688, 8064, 4096) > 0 and wsb(2688, 8064, 4000) == 0 and wsb(96, 8064, 4096) == 0
    assert wsb(2688, 8060, 4096) == 0
    # The workspace holds two BF16 x slots, one chunk of codes and MMA-tiled
    # scales, and two BF16 y slots, each padded to 256 bytes at most.
    for K, N, chunk in [(2688, 8064, 4096), (64, 8, 128), (2688, 10752, 1024), (10752, 2688, 384), (192, 24, 256)]:
        raw = 2 * chunk * K * 2 + chunk * K // 2 + -(-chunk // 128) * 128 * -(-(K // 16) // 4) * 4 + 2 * chunk * N * 2
        assert raw <= wsb(K, N, chunk) <= raw + 6 * 255, (K, N, chunk)
    need = wsb(2688, 8064, 4096)
    ws = P(1 << 20)  # a 256-byte-aligned fake address (never dereferenced here)
    assert hl(fake, 128, 2688, 1.0, fake, fake, 1.0, None, 8064, fake, None, 4000, ws, need, None) == 2  # chunk % 128
    assert hl(fake, 128, 2688, 1.0, fake, fake, 1.0, None, 8064, fake, None, 4096, ws, need - 1, None) == 1
    assert hl(fake, 128, 2688, 0.0, fake, fake, 1.0, None, 8064, fake, None, 4096, ws, need, None) == 1
    assert hl(None, 128, 2688, 1.0, fake, fake, 1.0, None, 8064, fake, None, 4096, ws, need, None) == 1
    assert hl(fake, 128, 2688, 1.0, fake, fake, 1.0, None, 8064, fake, None, 4096, P((1 << 20) + 16), need,
              None) == 2  # workspace alignment
    assert hl(fake, 0, 2688, 1.0, fake, fake, 1.0, None, 8064, fake, None, 4096, ws, need, None) == 0   # empty
    a = lib.fh_amax
    a.argtypes = [P, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, P, P]
    assert a(fake, 3, 5, 4, fake, None) == 2
    assert a(fake, 0, 5, 5, fake, None) == 0
    assert a(fake, 3, 5, 5, None, None) == 1


def test_package_refuses_to_import_without_library(tmp_path):
    """The binding fails loudly (no CPU fallback) when libfh.so is absent."""
    import shutil
    import subprocess
    import sys
    pkg = os.path.join(ROOT, "nvfp4_quantized_linear_fh_b200")
    dst = tmp_path / "nvfp4_quantized_linear_fh_b200"
    shutil.copytree(pkg, dst, ignore=shutil.ignore_patterns("*.so", "__pycache__", "csrc"))
    r = subprocess.run([sys.executable, "-c", "import nvfp4_quantized_linear_fh_b200"], cwd=tmp_path,
                       capture_output=True, text=True)
    assert r.returncode != 0 and "no CPU fallback" in r.stderr
