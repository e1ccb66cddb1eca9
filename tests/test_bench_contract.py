"""The benchmark's output contract, checked on the CPU: the reference arm (the
oracle timed on host cores) prints one JSON line with every key the contract
names, and the algorithmic byte counts the roofline divides by match the
formats' sizes."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference"
    assert line["steps"] == 1 and line["warmup"] == 3 and line["n_gpus"] == 1
    assert line["value"] > 0 and line["higher_is_better"] is True
    assert line["config"]["workload"].startswith("fused QKV linear 32768x2688->8064")
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["e2e"]["value"] == line["value"]


def test_algorithmic_bytes():
    M, K, N = 32768, 2688, 8064
    # A codes (K/2 bytes per row) and scales (K/16), the same for W, BF16 bias and y.
    assert bench.gemm_bytes(M, N, K) == M * K // 2 + M * K // 16 + N * K // 2 + N * K // 16 + 2 * N + 2 * M * N
    assert bench.gemm_bytes(M, N, K) == 590236416
    # INT8 scores: Q and K codes plus FP32 scales, FP32 S.
    assert bench.attn_score_bytes(21, 4096, 4096, 128) == 21 * 8192 * 132 + 4 * 21 * 4096 * 4096
    # Per-row INT8 quantization: BF16 in, INT8 out, one FP32 scale.
    assert bench.attn_quant_bytes(10, 128) == 10 * (3 * 128 + 4)
    # AdaLN: embeddings, basis, projections and biases in; codes and modulations out.
    assert bench.adaln_bytes(42, 16128, 2688, 16, 8) == 44836352
