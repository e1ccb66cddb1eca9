"""Benchmark of the NVFP4 quantized linear layer on B200.

One step = one pass of the whole hot path over one batch: NVFP4 quantization
of the BF16 activations with the layer's calibrated scale (fh_quantize_act)
followed by the block-scaled tensor-core GEMM with its fused epilogue
(fh_nvfp4_linear), on the fused-QKV workload of the transformer (FastH3 Trim,
comfyui-wiki news: hidden width 2688): M = 32768 tokens, K = 2688, N = 8064.
The calibration, the weight quantization and the input generation happen
before the timed region.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fh|reference]
  python bench.py --workload ffn|attn|adaln   (the FFN block, INT8 attention
      scores and AdaLN basis projection, one GPU; secondary lines)

With N > 1 (launched by torch.distributed.run) every rank runs the same
per-GPU workload on its own GPU (rows of the token batch are independent:
weak scaling, no data-path collective); the time is the max over ranks.
--impl reference times the CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4 linear TFLOPS (M×2688→N) and % of B200 FP4 peak; quantizer GB/s"
WORKLOAD = {"name": "qkv", "M": 32768, "K": 2688, "N": 8064}
FP4_OVER_BF16 = 4.0        # nominal dense ratio 9 / 2.25 PFLOP/s
QUANT_BYTES_PER_ELEM = 2.0 + 0.5 + 1.0 / 16.0
CPU_SAMPLE_ROWS = 8192   # about 13 s of the oracle on 16 host cores
# DRAM bytes (read + write) of one GEMM launch on this workload, from an ncu
# capture (dram__bytes_read.sum + dram__bytes_write.sum); valid only for the
# kernel source it was taken on (first 16 hex digits of its SHA-256).
GEMM_TRAFFIC = {"bytes": 576101376, "source_sha256": "4abe7c48fa84e050"}
# The same for one quantizer launch inside the step (ncu --cache-control none,
# so the L2 state the preceding GEMM left is kept); fh_quant.cu's hash.
QUANT_TRAFFIC = {"bytes": 231934336, "source_sha256": "2c5a04f54e2905b2"}
REF_ROWS = 16


def _traffic(record, source):
    """A recorded per-launch DRAM traffic figure if the kernel source is the one it was measured on."""
    import hashlib
    path = os.path.join(ROOT, "nvfp4_quantized_linear_fh_b200", "csrc", source)
    with open(path, "rb") as f:
        digest = hashlib.sha256(f.read()).hexdigest()[:16]
    return record["bytes"] if digest == record["source_sha256"] else None


def gemm_traffic():
    return _traffic(GEMM_TRAFFIC, "fh_gemm.cu")


def quant_traffic():
    return _traffic(QUANT_TRAFFIC, "fh_quant.cu")


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16": p["bf16_tflops"], "bf16_sustained": p["bf16_tflops_sustained"],
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id
        self.proc = None
        self.lines = []          # (host time, csv line)
        self.t0 = self.t1 = None

    def wait_first_sample(self, timeout: float = 3.0):
        end = time.time() + timeout
        while self.proc is not None and not self.lines and time.time() < end:
            time.sleep(0.01)

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()
        time.sleep(0.05)         # one more sample interval

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "10"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, pw, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        # samples taken while the timed region ran (nvidia-smi reports each sample
        # shortly after it is taken, so allow one interval of slack at the end)
        lo, hi = (self.t0 or 0.0), (self.t1 or 1e30) + 0.04
        window = [l for t, l in self.lines if lo <= t <= hi]
        for line in window:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
                pw.append(float(parts[3]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "power_w": statistics.median(pw) if pw else None, "samples": len(sm), "interval_ms": 10}


def make_inputs(rank: int, M: int, quick: bool):
    """Seeded synthetic fused-QKV layer (channel std log-normal, calibration over
    1000 batches of 64 tokens whose first M/64 form the input)."""
    import synthetic as S
    layer = S.workloads()["qkv"][0]
    n_calib = M // layer.batch if quick else max(layer.n_calib, M // layer.batch)
    layer = S.Layer(layer.name, M, layer.K, layer.N, layer.batch, n_calib, channel_lognormal=True,
                    key=layer.key if rank == 0 else ("qkv", rank))
    return S, layer


def bench_fh(args, rank, world, local_rank):
    import torch
    import nvfp4_quantized_linear_fh_b200 as fh

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    S, layer = make_inputs(rank, args.M, args.quick)
    M, K, N = layer.M, layer.K, layer.N

    # --- offline: inputs drawn on the GPU, calibration, weight quantization (not timed) ---
    x, sg_a = _dev_inputs(fh, S, layer, M, dev, calib=layer.n_calib)
    wc, wsc, sg_w, bias, w = _dev_weights(fh, S, layer, dev)
    x_bits, w_bits, b_bits = _bits(x[:CPU_SAMPLE_ROWS]), _bits(w), _bits(bias)
    del w

    ac, asc = fh.empty_quantized(M, K, device=dev)
    clip = torch.zeros(1, dtype=torch.int64, device=dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        fh.fh_quantize_act(x, sg_a, ac, asc, clip)
        fh.fh_nvfp4_linear(ac, asc, sg_a, wc, wsc, sg_w, bias, y)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clip.zero_()

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(f"GPU-{torch.cuda.get_device_properties(dev).uuid}")
    with sampler:
        sampler.wait_first_sample()
        sampler.mark_start()
        for i in range(args.steps):
            ev[i][0].record(stream)
            fh.fh_quantize_act(x, sg_a, ac, asc, clip)
            ev[i][1].record(stream)
            fh.fh_nvfp4_linear(ac, asc, sg_a, wc, wsc, sg_w, bias, y)
            ev[i][2].record(stream)
        torch.cuda.synchronize()
        sampler.mark_end()
    if world > 1:
        torch.distributed.barrier()
    t_quant = [ev[i][0].elapsed_time(ev[i][1]) * 1e-3 for i in range(args.steps)]
    t_gemm = [ev[i][1].elapsed_time(ev[i][2]) * 1e-3 for i in range(args.steps)]
    t_step = sum(t_quant) + sum(t_gemm)
    fh.fh_device_status()
    clips = int(clip.item())

    # --- the quantization fused into the GEMM (one launch), timed the same way ---
    t_fused = []
    if not args.no_fused:
        sync = fh.empty_fused_sync(M, device=dev)
        yf = torch.empty_like(y)
        acf, ascf = fh.empty_quantized(M, K, device=dev)
        for _ in range(args.warmup):
            fh.fh_nvfp4_linear_fused_quant(x, sg_a, wc, wsc, sg_w, bias, yf, acf, ascf, None, sync)
        torch.cuda.synchronize()
        fev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(min(args.steps, 50))]
        for e in fev:
            e[0].record(stream)
            fh.fh_nvfp4_linear_fused_quant(x, sg_a, wc, wsc, sg_w, bias, yf, acf, ascf, None, sync)
            e[1].record(stream)
        torch.cuda.synchronize()
        fh.fh_device_status()
        t_fused = [e[0].elapsed_time(e[1]) * 1e-3 for e in fev]
        if not torch.equal(yf.view(torch.int16), y.view(torch.int16)):
            raise RuntimeError("the fused path's output differs from the two separate calls")
        del sync, yf, acf, ascf

    # --- end to end through the public API with host buffers ---
    # fh_nvfp4_linear_host: pinned BF16 x in host memory -> BF16 y in host
    # memory, the upload, kernels and download pipelined over 4096-row chunks.
    t_e2e, e_steps = float('nan'), 0
    if not args.no_e2e:
        x_host = torch.empty((M, K), dtype=torch.bfloat16, pin_memory=True)
        x_host.copy_(x.cpu())
        y_host = torch.empty((M, N), dtype=torch.bfloat16, pin_memory=True)
        chunk = 4096
        ws = torch.empty(fh.fh_nvfp4_linear_host_workspace_bytes(K, N, chunk), dtype=torch.uint8, device=dev)
        e_steps = max(2, min(args.steps, 5))
        for _ in range(2):
            fh.fh_nvfp4_linear_host(x_host, sg_a, wc, wsc, sg_w, bias, y_host, None, chunk, ws)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            torch.distributed.barrier()
        e0.record(stream)
        for _ in range(e_steps):
            fh.fh_nvfp4_linear_host(x_host, sg_a, wc, wsc, sg_w, bias, y_host, None, chunk, ws)
        e1.record(stream)
        torch.cuda.synchronize()
        t_e2e = e0.elapsed_time(e1) * 1e-3
        del ws

    if world > 1:
        from nvfp4_quantized_linear_fh_b200 import dist as fhd
        t_step, t_e2e = fhd.max_over_ranks([t_step, t_e2e], device=dev)
    flops = 2.0 * M * N * K
    return dict(t_step=t_step, t_quant=t_quant, t_gemm=t_gemm, t_e2e=t_e2e, e_steps=e_steps, flops=flops, t_fused=t_fused,
                clips=clips, sampler=sampler.summary(), M=M, N=N, K=K,
                h2d=M * K * 2, d2h=M * N * 2, x_bits=x_bits, w_bits=w_bits, b_bits=b_bits,
                sg_a=sg_a, sg_w=sg_w)


_WQ_CACHE = {}


def fp4_tensor_rate(with_copies: bool, iters: int = 60000, reps: int = 3) -> float:
    """FLOP/s of the library's tensor-rate probe: every CTA pair issues `iters`
    rounds of four 256 x 256 x 64 block-scaled FP4 MMAs from shared memory
    (with_copies: plus the GEMM's twelve scale copies per round), timed with
    CUDA events; the best of `reps` launches after a warm-up."""
    import torch
    import nvfp4_quantized_linear_fh_b200 as fh
    fh.fh_selftest_mma_rate(2000, with_copies)
    best = 0.0
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        pairs = fh.fh_selftest_mma_rate(iters, with_copies)
        e1.record()
        torch.cuda.synchronize()
        best = max(best, pairs * iters * 2.0 * 256 ** 3 / (e0.elapsed_time(e1) * 1e-3))
    fh.fh_device_status()
    return best


def gemm_bytes(M, N, K):
    """Algorithmic bytes of one GEMM launch: A and W codes and scales, bias, BF16 output."""
    return M * K // 2 + M * K // 16 + N * K // 2 + N * K // 16 + 2 * N + 2 * M * N


def cpu_baseline(x_bits, w_bits, b_bits, sg_a, sg_w, rows):
    """The oracle, as it stands, on the first `rows` token rows of one step:
    quantize those activation rows and run the binary64 dequantized product
    against the weights (quantized once beforehand, like the GPU path's
    offline weights).  Returns (TFLOPS, seconds, cores)."""
    import oracle
    oracle.build()
    K, N = x_bits.shape[1], w_bits.shape[0]
    key = (id(w_bits), sg_w)
    if key not in _WQ_CACHE:
        _WQ_CACHE[key] = oracle.quantize(w_bits, sg_w)[:2]
    wc, wsc = _WQ_CACHE[key]
    t0 = time.perf_counter()
    ac, asc, _ = oracle.quantize(x_bits[:rows], sg_a)
    oracle.linear(ac, asc, sg_a, wc, wsc, sg_w, b_bits)
    dt = time.perf_counter() - t0
    cores = len(os.sched_getaffinity(0))
    return 2.0 * rows * N * K / dt / 1e12, dt, cores


def bench_ffn(args):
    """The FFN block of the 2688-wide transformer (up 2688->10752, GELU, down
    10752->2688) on args.M tokens, timed two ways on the same operands:
    unfused (quantize, GEMM, GELU, quantize, GEMM) and fused (quantize, GEMM
    whose epilogue applies GELU and quantizes for the down projection, GEMM)."""
    import torch
    import synthetic as S
    import nvfp4_quantized_linear_fh_b200 as fh

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    up, down = S.workloads()["ffn"]
    M, K, N1 = args.M, up.K, up.N
    N2 = down.N

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)

    def quant_weight(layer):
        w = to_dev(S.weights(layer))
        wamax = torch.zeros(1, dtype=torch.float32, device=dev)
        fh.fh_amax(w, wamax)
        sg = fh.fh_scale_from_amax(wamax.item())
        wc, wsc = fh.empty_quantized(layer.N, layer.K, device=dev)
        fh.fh_quantize_act(w, sg, wc, wsc, None)
        return wc, wsc, sg, to_dev(S.bias(layer))

    import dataclasses
    x = to_dev(S.activations(dataclasses.replace(up, M=M, n_calib=max(up.n_calib, M // up.batch))))
    w1c, w1s, sg_w1, b1 = quant_weight(up)
    w2c, w2s, sg_w2, b2 = quant_weight(down)
    amax = torch.zeros(1, dtype=torch.float32, device=dev)
    fh.fh_amax(x, amax)
    sg_x = fh.fh_scale_from_amax(amax.item())
    xc, xs = fh.empty_quantized(M, K, device=dev)
    y1 = torch.empty((M, N1), dtype=torch.bfloat16, device=dev)
    g = torch.empty_like(y1)
    gc, gs = fh.empty_quantized(M, N1, device=dev)
    out = torch.empty((M, N2), dtype=torch.bfloat16, device=dev)
    # Down-projection input scale: calibrated on the GELU output of this input.
    fh.fh_quantize_act(x, sg_x, xc, xs, None)
    fh.fh_nvfp4_linear(xc, xs, sg_x, w1c, w1s, sg_w1, b1, y1)
    fh.fh_gelu_bf16(y1, g)
    amax.zero_()
    fh.fh_amax(g, amax)
    sg_g = fh.fh_scale_from_amax(amax.item())

    def unfused():
        fh.fh_quantize_act(x, sg_x, xc, xs, None)
        fh.fh_nvfp4_linear(xc, xs, sg_x, w1c, w1s, sg_w1, b1, y1)
        fh.fh_gelu_bf16(y1, g)
        fh.fh_quantize_act(g, sg_g, gc, gs, None)
        fh.fh_nvfp4_linear(gc, gs, sg_g, w2c, w2s, sg_w2, b2, out)

    def gelu_quant():
        fh.fh_quantize_act(x, sg_x, xc, xs, None)
        fh.fh_nvfp4_linear(xc, xs, sg_x, w1c, w1s, sg_w1, b1, y1)
        fh.fh_gelu_quantize_act(y1, sg_g, gc, gs, None)
        fh.fh_nvfp4_linear(gc, gs, sg_g, w2c, w2s, sg_w2, b2, out)

    def fused():
        fh.fh_quantize_act(x, sg_x, xc, xs, None)
        fh.fh_nvfp4_linear_gelu_quant(xc, xs, sg_x, w1c, w1s, sg_w1, b1, sg_g, gc, gs, None)
        fh.fh_nvfp4_linear(gc, gs, sg_g, w2c, w2s, sg_w2, b2, out)

    def timed(fn, steps):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) * 1e-3 / steps

    steps = max(1, min(args.steps, 100))
    variants = {"unfused": (unfused, "quantize, linear, gelu, quantize, linear"),
                "gelu_quant": (gelu_quant, "quantize, linear, gelu_quantize, linear"),
                "fused_epilogue": (fused, "quantize, linear_gelu_quant, linear")}
    times, identical, ref_out = {}, True, None
    for name, (fn, _) in variants.items():
        times[name] = timed(fn, steps)
        if ref_out is None:
            ref_out = out.clone()
        else:
            identical = identical and bool(torch.equal(out.view(torch.int16), ref_out.view(torch.int16)))
    fh.fh_device_status()
    flops = 2.0 * M * K * N1 + 2.0 * M * N1 * N2
    best = min(times, key=times.get)
    print(json.dumps({
        "metric": "NVFP4 FFN block TFLOPS (up 2688->10752, GELU, down 10752->2688)", "unit": "TFLOPS",
        "value": flops / times[best] / 1e12, "ms_per_step": times[best] * 1e3, "best": best, "steps": steps,
        "warmup": args.warmup, "n_gpus": 1, "higher_is_better": True,
        "data": "synthetic (seeded; random-init weights)",
        "config": {"workload": f"FFN block {M}x2688->10752->2688 per GPU", "M": M},
        "variants": {n: {"value": flops / t / 1e12, "ms_per_step": t * 1e3, "calls": variants[n][1]}
                     for n, t in times.items()},
        "outputs_bit_identical": identical}))


# ---------------------------------------------------------------------------
# The five synthetic configurations, each with its own roofline fractions and
# its oracle baseline (the "configs" object of the default line, or one line
# each with --workload tiny|attn_proj|ffn_pair|block_sweep).
# ---------------------------------------------------------------------------

def _dev_inputs(fh, S, layer, M, dev, calib):
    """The layer's first M rows (BF16, drawn on the GPU) and its calibrated global scale:
    amax over `calib` batches of its calibration stream (the input being their prefix)."""
    import torch
    nb = M // layer.batch
    x = S.activation_batches_t(layer, 0, nb, dev).view(torch.bfloat16)
    amax = torch.zeros(1, dtype=torch.float32, device=dev)
    fh.fh_amax(x, amax)
    for b0 in range(nb, calib, 128):
        n = min(128, calib - b0)
        fh.fh_amax(S.activation_batches_t(layer, b0, n, dev).view(torch.bfloat16), amax)
    return x, fh.fh_scale_from_amax(amax.item())


def _dev_weights(fh, S, layer, dev):
    """W drawn on the GPU and quantized offline with its own amax scale; the BF16 W is returned too."""
    import torch
    w = S.weights_t(layer, dev).view(torch.bfloat16)
    wamax = torch.zeros(1, dtype=torch.float32, device=dev)
    fh.fh_amax(w, wamax)
    sg = fh.fh_scale_from_amax(wamax.item())
    wc, wsc = fh.empty_quantized(layer.N, layer.K, device=dev)
    fh.fh_quantize_act(w, sg, wc, wsc, None)
    return wc, wsc, sg, S.bias_t(layer, dev).view(torch.bfloat16), w


def _bits(t):
    return t.view(__import__("torch").int16).cpu().numpy().view(np.uint16)


def _time_calls(calls, steps, warmup, flush=None):
    """calls: [(tag, fn)] making one step.  Runs `warmup` untimed steps, then
    `steps` steps with a CUDA event between consecutive calls (and `flush`, if
    given, before each step, outside the events).  Returns ({tag: seconds per
    step, summed over the tag's calls}, seconds of the whole timed region)."""
    import torch
    for _ in range(warmup):
        if flush is not None:
            flush()
        for _, fn in calls:
            fn()
    torch.cuda.synchronize()
    evs = []
    for _ in range(steps):
        if flush is not None:
            flush()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)]
        ev[0].record()
        for i, (_, fn) in enumerate(calls):
            fn()
            ev[i + 1].record()
        evs.append(ev)
    torch.cuda.synchronize()
    out = {}
    for ev in evs:
        for i, (tag, _) in enumerate(calls):
            out[tag] = out.get(tag, 0.0) + ev[i].elapsed_time(ev[i + 1]) * 1e-3
    region = sum(out.values())
    return {k: v / steps for k, v in out.items()}, region


def _gemm_roof(flops, secs, pk, sustained):
    burst, sust = pk["bf16"] * FP4_OVER_BF16, pk["bf16_sustained"] * FP4_OVER_BF16
    ach = flops / secs / 1e12
    peak = sust if sustained else burst
    return {"bound": "tensor", "achieved": ach, "unit": "TFLOP/s", "peak": peak, "frac": ach / peak,
            "peak_kind": "sustained" if sustained else "burst", "frac_of_burst_peak": ach / burst,
            "frac_of_sustained_peak": ach / sust}


def _quant_roof(M, K, secs, pk):
    ach = QUANT_BYTES_PER_ELEM * M * K / secs / 1e9
    return {"bound": "hbm", "achieved": ach, "unit": "GB/s", "peak": pk["hbm_gbs"], "frac": ach / pk["hbm_gbs"],
            "us": secs * 1e6}


def _oracle_layer_rate(x_bits, sg_a, wq, b_bits, rows):
    """The oracle on `rows` token rows: quantize them, binary64 dequantized GEMM
    against the already-quantized weights wq = (codes, scales, s_gW).
    Returns (FLOP/s, seconds)."""
    import oracle
    wc, wsc, sg_w = wq
    K, N = x_bits.shape[1], wc.shape[0]
    t0 = time.perf_counter()
    ac, asc, _ = oracle.quantize(x_bits[:rows], sg_a)
    oracle.linear(ac, asc, sg_a, wc, wsc, sg_w, b_bits)
    dt = time.perf_counter() - t0
    return 2.0 * rows * N * K / dt, dt


def _oracle_weights(w):
    import oracle
    wb = _bits(w)
    sg = oracle.scale_from_amax(oracle.amax(wb))
    c, s, _ = oracle.quantize(wb, sg)
    return c, s, sg


def measure_layer_config(name, fh, S, dev, pk, args):
    """tiny (128 x 256 -> 256) or attn_proj (8192 x 2688 -> 2688): quantize + GEMM per
    step; both fit in L2, so L2 is flushed (a 256 MB write) before every step."""
    import torch
    layer = S.workloads()[name][0]
    M, K, N = layer.M, layer.K, layer.N
    # Both recipes put one outlier of exactly 137 L in every batch, so the amax
    # over the evaluation batches is the amax over the whole calibration stream.
    x, sg_a = _dev_inputs(fh, S, layer, M, dev, calib=layer.n_eval_batches)
    wc, wsc, sg_w, b, w = _dev_weights(fh, S, layer, dev)
    ac, asc = fh.empty_quantized(M, K, device=dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    clip = torch.zeros(1, dtype=torch.int64, device=dev)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    calls = [("quant", lambda: fh.fh_quantize_act(x, sg_a, ac, asc, clip)),
             ("gemm", lambda: fh.fh_nvfp4_linear(ac, asc, sg_a, wc, wsc, sg_w, b, y))]
    steps = 100
    t, region = _time_calls(calls, steps, max(args.warmup, 3), flush=lambda: flush.fill_(1.0))
    fh.fh_device_status()
    flops = 2.0 * M * N * K
    out = {"workload": f"{name} {M}x{K}->{N}", "M": M, "K": K, "N": N, "steps": steps,
           "step_us": (t["quant"] + t["gemm"]) * 1e6, "tflops": flops / (t["quant"] + t["gemm"]) / 1e12,
           "gemm_us": t["gemm"] * 1e6, "gemm_roofline": _gemm_roof(flops, t["gemm"], pk, False),
           "quantizer_roofline": _quant_roof(M, K, t["quant"], pk), "clip_count": int(clip.item()),
           "l2": "flushed before every step (256 MB write, outside the timed events)"}
    if not args.no_cpu_baseline:
        rows = M if M <= 128 else 32
        rate, dt = _oracle_layer_rate(_bits(x), sg_a, _oracle_weights(w), _bits(b), rows)
        out["cpu_baseline"] = {"value": rate / 1e12, "unit": "TFLOPS", "cores": len(os.sched_getaffinity(0)),
                               "kind": "oracle", "sample": f"{rows} of the {M} token rows ({dt:.2f} s)"}
    return out


def measure_ffn_config(fh, S, dev, pk, args):
    """Config 4, the FFN pair at 32768 tokens: up 2688 -> 10752, GELU, down 10752 -> 2688,
    each layer's input quantized with its own calibrated scale (the down layer's
    calibrated on the GELU outputs of the same batches).  Two paths on the same
    operands: the plain chain (quantize, GEMM, GELU, quantize, GEMM) and the fused
    one (quantize, GEMM with the GELU-quantizing epilogue, GEMM)."""
    import torch
    up, down = S.workloads()["ffn"]
    M, K, N1, N2 = up.M, up.K, up.N, down.N
    # The up layer's recipe has one outlier of exactly 137 L per batch: the amax
    # over the evaluation batches is that of the whole stream.
    x, sg_x = _dev_inputs(fh, S, up, M, dev, calib=up.n_eval_batches)
    w1c, w1s, sg_w1, b1, w1 = _dev_weights(fh, S, up, dev)
    w2c, w2s, sg_w2, b2, w2 = _dev_weights(fh, S, down, dev)
    xc, xs = fh.empty_quantized(M, K, device=dev)
    h = torch.empty((M, N1), dtype=torch.bfloat16, device=dev)
    g = torch.empty_like(h)
    gc, gs = fh.empty_quantized(M, N1, device=dev)
    y = torch.empty((M, N2), dtype=torch.bfloat16, device=dev)
    clip = torch.zeros(1, dtype=torch.int64, device=dev)
    fh.fh_quantize_act(x, sg_x, xc, xs, clip)
    fh.fh_nvfp4_linear(xc, xs, sg_x, w1c, w1s, sg_w1, b1, h)
    fh.fh_gelu_bf16(h, g)
    amax = torch.zeros(1, dtype=torch.float32, device=dev)
    fh.fh_amax(g, amax)
    sg_g = fh.fh_scale_from_amax(amax.item())
    plain = [("quant_up", lambda: fh.fh_quantize_act(x, sg_x, xc, xs, clip)),
             ("gemm_up", lambda: fh.fh_nvfp4_linear(xc, xs, sg_x, w1c, w1s, sg_w1, b1, h)),
             ("gelu", lambda: fh.fh_gelu_bf16(h, g)),
             ("quant_down", lambda: fh.fh_quantize_act(g, sg_g, gc, gs, clip)),
             ("gemm_down", lambda: fh.fh_nvfp4_linear(gc, gs, sg_g, w2c, w2s, sg_w2, b2, y))]
    fused = [("quant_up", lambda: fh.fh_quantize_act(x, sg_x, xc, xs, clip)),
             ("gemm_up_gelu_quant", lambda: fh.fh_nvfp4_linear_gelu_quant(xc, xs, sg_x, w1c, w1s, sg_w1, b1, sg_g,
                                                                         gc, gs, clip)),
             ("gemm_down", lambda: fh.fh_nvfp4_linear(gc, gs, sg_g, w2c, w2s, sg_w2, b2, y))]
    steps = 20
    tp, _ = _time_calls(plain, steps, max(args.warmup, 3))
    y_plain = y.clone()
    clip.zero_()
    tf, _ = _time_calls(fused, steps, max(args.warmup, 3))
    fh.fh_device_status()
    identical = bool(torch.equal(y.view(torch.int16), y_plain.view(torch.int16)))
    f_up, f_down = 2.0 * M * K * N1, 2.0 * M * N1 * N2
    t_plain, t_fused = sum(tp.values()), sum(tf.values())
    out = {"workload": f"FFN pair {M}x{K}->{N1} (GELU) ->{N2}", "M": M, "K": K, "N_up": N1, "N_down": N2,
           "steps": steps, "block_ms_plain": t_plain * 1e3, "block_ms_fused": t_fused * 1e3,
           "tflops_plain": (f_up + f_down) / t_plain / 1e12, "tflops_fused": (f_up + f_down) / t_fused / 1e12,
           "outputs_bit_identical": identical, "clip_count": int(clip.item()),
           "kernels_us_plain": {k: v * 1e6 for k, v in tp.items()},
           "kernels_us_fused": {k: v * 1e6 for k, v in tf.items()},
           "gemm_up_roofline": _gemm_roof(f_up, tp["gemm_up"], pk, False),
           "gemm_down_roofline": _gemm_roof(f_down, tp["gemm_down"], pk, False),
           "gemm_up_gelu_quant_roofline": _gemm_roof(f_up, tf["gemm_up_gelu_quant"], pk, False),
           "quantizer_up_roofline": _quant_roof(M, K, tp["quant_up"], pk),
           "quantizer_down_roofline": _quant_roof(M, N1, tp["quant_down"], pk),
           "l2": "not flushed: every step's inputs and outputs exceed L2"}
    if not args.no_cpu_baseline:
        rows = 16
        r1, d1 = _oracle_layer_rate(_bits(x), sg_x, _oracle_weights(w1), _bits(b1), rows)
        r2, d2 = _oracle_layer_rate(_bits(g), sg_g, _oracle_weights(w2), _bits(b2), rows)
        out["cpu_baseline"] = {"value": 2.0 * rows * (K * N1 + N1 * N2) / (d1 + d2) / 1e12, "unit": "TFLOPS",
                               "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
                               "sample": f"{rows} token rows through both layers ({d1 + d2:.2f} s)"}
    return out


def measure_sweep_config(fh, S, dev, pk, args):
    """Config 5: 42 blocks x {QKV 2688->8064, out 2688->2688, up 2688->10752,
    down 10752->2688} = 168 layers back to back at 49152 tokens, each with its own
    seeded weights, its own calibrated scale (amax over its 1000-batch stream)
    and its own BF16 input (77 GB in all, resident in HBM), quantized per layer.
    One step = the 168 quantize + GEMM pairs."""
    import torch
    sweep = S.workloads()["block_sweep"]
    M = sweep[0].M
    layers = []
    shapes = {}
    for layer in sweep:
        x, sg_a = _dev_inputs(fh, S, layer, M, dev, calib=layer.n_calib)
        wc, wsc, sg_w, b, w = _dev_weights(fh, S, layer, dev)
        del w
        key = (layer.K, layer.N)
        if key not in shapes:  # codes and outputs are per shape: each layer overwrites its shape's buffers
            shapes[key] = (*fh.empty_quantized(M, layer.K, device=dev),
                           torch.empty((M, layer.N), dtype=torch.bfloat16, device=dev))
        layers.append((layer, x, sg_a, wc, wsc, sg_w, b))
    clip = torch.zeros(1, dtype=torch.int64, device=dev)
    calls = []
    for (layer, x, sg_a, wc, wsc, sg_w, b) in layers:
        ac, asc, y = shapes[(layer.K, layer.N)]
        tag = f"{layer.K}->{layer.N}"
        calls.append(("quant " + tag, lambda x=x, sg_a=sg_a, ac=ac, asc=asc: fh.fh_quantize_act(x, sg_a, ac, asc, clip)))
        calls.append(("gemm " + tag, lambda ac=ac, asc=asc, sg_a=sg_a, wc=wc, wsc=wsc, sg_w=sg_w, b=b, y=y:
                      fh.fh_nvfp4_linear(ac, asc, sg_a, wc, wsc, sg_w, b, y)))
    steps = 3
    t, region = _time_calls(calls, steps, 3)
    fh.fh_device_status()
    nb = len(sweep) // 4
    flops = {f"{l.K}->{l.N}": 2.0 * M * l.K * l.N * nb for l in sweep[:4]}
    t_gemm = sum(v for k, v in t.items() if k.startswith("gemm"))
    t_quant = sum(v for k, v in t.items() if k.startswith("quant"))
    total_flops = sum(flops.values())
    quant_bytes = QUANT_BYTES_PER_ELEM * M * sum(l.K for l in sweep)
    # A 168-layer step runs for ~0.1 s of back-to-back GEMMs: the power-capped
    # (sustained) GEMM figure is its denominator.
    out = {"workload": f"block sweep {len(sweep)} layers at M={M}", "M": M, "layers": len(sweep), "steps": steps,
           "step_ms": (t_gemm + t_quant) * 1e3, "tflops": total_flops / (t_gemm + t_quant) / 1e12,
           "gemm_roofline": _gemm_roof(total_flops, t_gemm, pk, True),
           "quantizer_roofline": {"bound": "hbm", "achieved": quant_bytes / t_quant / 1e9, "unit": "GB/s",
                                  "peak": pk["hbm_gbs"], "frac": quant_bytes / t_quant / 1e9 / pk["hbm_gbs"],
                                  "us": t_quant * 1e6},
           "per_shape": {tag: {"gemm_us_per_layer": t["gemm " + tag] / nb * 1e6,
                               "gemm_tflops": flops[tag] / t["gemm " + tag] / 1e12,
                               "quant_us_per_layer": t["quant " + tag] / nb * 1e6,
                               "quant_gbs": QUANT_BYTES_PER_ELEM * M * int(tag.split("->")[0]) * nb
                               / t["quant " + tag] / 1e9} for tag in flops},
           "clip_count": int(clip.item()), "inputs_gb": 2.0 * M * sum(l.K for l in sweep) / 1e9,
           "l2": "not flushed: every layer's input (>= 264 MB) exceeds L2"}
    if not args.no_cpu_baseline:
        rows, secs, fl = 8, 0.0, 0.0
        for (layer, x, sg_a, wc, wsc, sg_w, b) in layers[:4]:
            w = S.weights_t(layer, dev).view(torch.bfloat16)
            r, dt = _oracle_layer_rate(_bits(x[:rows]), sg_a, _oracle_weights(w), _bits(b), rows)
            secs += dt
            fl += 2.0 * rows * layer.K * layer.N
        out["cpu_baseline"] = {"value": fl / secs / 1e12, "unit": "TFLOPS", "cores": len(os.sched_getaffinity(0)),
                               "kind": "oracle", "sample": f"{rows} token rows through block 0's four layers "
                                                           f"({secs:.2f} s)"}
    del layers, shapes
    torch.cuda.empty_cache()
    return out


def measure_configs(args, which=("tiny", "attn_proj", "ffn_pair", "block_sweep")):
    import torch
    import synthetic as S
    import nvfp4_quantized_linear_fh_b200 as fh
    dev = torch.device("cuda", torch.cuda.current_device())
    pk = peaks()
    out = {}
    for name in which:
        if name in ("tiny", "attn_proj"):
            out[name] = measure_layer_config(name, fh, S, dev, pk, args)
        elif name == "ffn_pair":
            out[name] = measure_ffn_config(fh, S, dev, pk, args)
        elif name == "block_sweep":
            out[name] = measure_sweep_config(fh, S, dev, pk, args)
        torch.cuda.empty_cache()
    return out


ATTN = {"heads": 21, "tokens": 4096, "d": 128}


def attn_score_bytes(H, tq, tk, d):
    """Algorithmic bytes of one score launch: INT8 Q and K, their FP32 scales, FP32 scores."""
    return H * (tq + tk) * (d + 4) + 4 * H * tq * tk


def attn_quant_bytes(rows, d):
    """Algorithmic bytes of one INT8 row-quantizer launch: BF16 in, INT8 codes and FP32 scales out."""
    return rows * (3 * d + 4)


def bench_attn(args):
    """INT8 attention scores of the 2688-wide transformer's self-attention
    (21 heads x d 128, 4096 queries x 4096 keys per head): per-row INT8
    quantization of Q and of K, then the tensor-core score kernel writing FP32
    S[h, i, j].  One step = quantize Q, quantize K, scores."""
    import torch
    import synthetic as S
    import nvfp4_quantized_linear_fh_b200 as fh

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    H, T, d = ATTN["heads"], ATTN["tokens"], ATTN["d"]

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)

    qb, kb = S.attention_qk(H, T, d, "q", 1), S.attention_qk(H, T, d, "k", 1)
    xq, xk = to_dev(qb.reshape(H * T, d)), to_dev(kb.reshape(H * T, d))
    q8 = torch.empty((H, T, d), dtype=torch.int8, device=dev)
    k8 = torch.empty_like(q8)
    qs = torch.empty((H, T), dtype=torch.float32, device=dev)
    ks = torch.empty_like(qs)
    sc = torch.empty((H, T, T), dtype=torch.float32, device=dev)
    sm_scale = float(np.float32(1.0 / np.sqrt(d)))
    stream = torch.cuda.current_stream()

    def step():
        fh.fh_quantize_int8_rows(xq, q8.view(H * T, d), qs.view(-1))
        fh.fh_quantize_int8_rows(xk, k8.view(H * T, d), ks.view(-1))
        fh.fh_int8_attention_scores(q8, qs, k8, ks, sm_scale, sc)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    steps = max(1, min(args.steps, 200))
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    sampler = ClockSampler(f"GPU-{torch.cuda.get_device_properties(dev).uuid}")
    with sampler:
        sampler.wait_first_sample()
        sampler.mark_start()
        for i in range(steps):
            ev[i][0].record(stream)
            fh.fh_quantize_int8_rows(xq, q8.view(H * T, d), qs.view(-1))
            fh.fh_quantize_int8_rows(xk, k8.view(H * T, d), ks.view(-1))
            ev[i][1].record(stream)
            fh.fh_int8_attention_scores(q8, qs, k8, ks, sm_scale, sc)
            ev[i][2].record(stream)
        torch.cuda.synchronize()
        sampler.mark_end()
    fh.fh_device_status()
    t_quant = sum(ev[i][0].elapsed_time(ev[i][1]) for i in range(steps)) * 1e-3 / steps
    t_scores = sum(ev[i][1].elapsed_time(ev[i][2]) for i in range(steps)) * 1e-3 / steps
    t_step = t_quant + t_scores
    ops = 2.0 * H * T * T * d

    # End to end: BF16 Q and K from pinned host memory, FP32 scores back to pinned host memory.
    t_e2e, e_steps = float("nan"), 0
    if not args.no_e2e:
        xq_h = torch.empty_like(xq, device="cpu").pin_memory()
        xk_h = torch.empty_like(xk, device="cpu").pin_memory()
        xq_h.copy_(xq.cpu())
        xk_h.copy_(xk.cpu())
        s_h = torch.empty((H, T, T), dtype=torch.float32).pin_memory()
        e_steps = 3
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(e_steps):
            xq.copy_(xq_h, non_blocking=True)
            xk.copy_(xk_h, non_blocking=True)
            step()
            s_h.copy_(sc, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        t_e2e = e0.elapsed_time(e1) * 1e-3 / e_steps

    pk = peaks()
    by = attn_score_bytes(H, T, T, d)
    achieved = by / t_scores / 1e9
    line = {
        "metric": "INT8 attention scores: whole-step TOPS (quantize Q, quantize K, Q.K^T scaled to FP32)",
        "value": ops / t_step / 1e12, "unit": "TOPS", "n_gpus": 1, "steps": steps, "warmup": args.warmup,
        "ms_per_step": t_step * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "s8 (INT32 accumulate, FP32 scores)", "data": "synthetic (seeded Q/K with outlier channels)",
        "config": {"workload": f"attention scores {H} heads x {T} queries x {T} keys x d {d}", "heads": H,
                   "tq": T, "tk": T, "d": d,
                   "l2": "not flushed: each step writes 1.41 GB of scores (> L2)"},
        "kernels_us": {"int8_quantize_rows (Q and K)": t_quant * 1e6, "int8_scores_kernel": t_scores * 1e6},
        "roofline": {"bound": "hbm", "kernel": "int8_scores_kernel", "achieved": achieved, "peak": pk["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved / pk["hbm_gbs"], "peak_source": pk["source"],
                     "traffic": ATTN_TRAFFIC["bytes"] if attn_traffic_valid() else None,
                     "algorithmic_bytes": by},
        "quantizer": {"achieved_gbs": 2 * attn_quant_bytes(H * T, d) / t_quant / 1e9},
        "e2e": {"value": ops / t_e2e / 1e12 if e_steps else None, "unit": "TOPS",
                "h2d_bytes_per_step": 2 * H * T * d * 2, "d2h_bytes_per_step": 4 * H * T * T},
        "gpu_launches": 3 * steps, "clocks": sampler.summary(),
    }
    if not args.no_cpu_baseline:
        import oracle
        rows = T  # one whole head: a few seconds of oracle work
        t0 = time.perf_counter()
        oq, oqs = oracle.quantize_int8_rows(qb[0, :rows])
        ok, oks = oracle.quantize_int8_rows(kb[0])
        oracle.int8_scores(oq[None], oqs[None], ok[None], oks[None], sm_scale)
        dt = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": 2.0 * rows * T * d / dt / 1e12, "unit": "TOPS",
                                "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
                                "sample": f"head 0 of {H}: its {rows} query and {T} key rows quantized, "
                                          f"their {rows}x{T} scores"}
    print(json.dumps(line))


ADALN = {"blocks": 42, "n": 6 * 2688, "d": 2688, "r": 16}


def adaln_bytes(blocks, n, d, r, bt):
    """Algorithmic bytes of one fh_adaln_modulation call: embeddings, basis, projections
    and biases read once; codes and modulations written once."""
    return 2 * bt * d + 2 * r * d + 2 * blocks * n * r + 2 * blocks * n + 4 * bt * r + 4 * blocks * bt * n


def bench_adaln(args):
    """AdaLN timestep conditioning of the 42-block pruned transformer: the eight
    sampler timesteps' 2688-wide embeddings through the shared 2688->16 basis and
    each block's 16->6*2688 projection (FP16 weights, FP32 results).  The inputs
    (45 MB) fit in L2, so L2 is flushed (a 256 MB write) before every timed call."""
    import torch
    import synthetic as S
    import nvfp4_quantized_linear_fh_b200 as fh

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    L, n, d, r = ADALN["blocks"], ADALN["n"], ADALN["d"], ADALN["r"]
    ts = S.SAMPLER_TIMESTEPS
    bt = len(ts)
    e_b, basis_b, proj_b, bias_b = S.adaln_inputs(L, n, d, r, ts)

    def to_dev(bits, dtype):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(dtype)

    e, basis = to_dev(e_b, torch.bfloat16), to_dev(basis_b, torch.float16)
    proj, bias = to_dev(proj_b, torch.float16), to_dev(bias_b, torch.float16)
    code = torch.empty((bt, r), dtype=torch.float32, device=dev)
    mod = torch.empty((L, bt, n), dtype=torch.float32, device=dev)
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)  # 256 MB > L2
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        fh.fh_adaln_modulation(e, basis, proj, bias, code, mod)
    torch.cuda.synchronize()
    steps = max(1, min(args.steps, 500))
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    sampler = ClockSampler(f"GPU-{torch.cuda.get_device_properties(dev).uuid}")
    with sampler:
        sampler.wait_first_sample()
        sampler.mark_start()
        for i in range(steps):
            flush.fill_(float(i))
            ev[i][0].record(stream)
            fh.fh_adaln_modulation(e, basis, proj, bias, code, mod)
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        sampler.mark_end()
    fh.fh_device_status()
    t = sum(ev[i][0].elapsed_time(ev[i][1]) for i in range(steps)) * 1e-3 / steps
    by = adaln_bytes(L, n, d, r, bt)

    t_e2e, e_steps = float("nan"), 0
    if not args.no_e2e:
        e_h = torch.empty(e.shape, dtype=torch.bfloat16).pin_memory()
        e_h.copy_(e.cpu())
        mod_h = torch.empty(mod.shape, dtype=torch.float32).pin_memory()
        e_steps = 20
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(e_steps):
            e.copy_(e_h, non_blocking=True)
            fh.fh_adaln_modulation(e, basis, proj, bias, code, mod)
            mod_h.copy_(mod, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        t_e2e = e0.elapsed_time(e1) * 1e-3 / e_steps

    pk = peaks()
    line = {
        "metric": "AdaLN basis projection: GB/s of algorithmic HBM traffic per call (8 timesteps x 42 blocks)",
        "value": by / t / 1e9, "unit": "GB/s", "n_gpus": 1, "steps": steps, "warmup": args.warmup,
        "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32 (FP16 weights, BF16 embeddings)", "data": "synthetic (seeded; random-init weights)",
        "config": {"workload": f"AdaLN modulation {bt} timesteps x {L} blocks x {n} (d {d}, rank {r})",
                   "blocks": L, "n": n, "d": d, "r": r, "timesteps": bt,
                   "l2": "flushed before every timed call (256 MB write, outside the timed events)"},
        "roofline": {"bound": "hbm", "kernel": "adaln_code_kernel + adaln_mod_kernel (one call)",
                     "achieved": by / t / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": by / t / 1e9 / pk["hbm_gbs"], "peak_source": pk["source"], "traffic": None,
                     "algorithmic_bytes": by},
        "e2e": {"value": by / t_e2e / 1e9 if e_steps else None, "unit": "GB/s",
                "h2d_bytes_per_step": 2 * bt * d, "d2h_bytes_per_step": 4 * L * bt * n},
        "gpu_launches": 2 * steps, "clocks": sampler.summary(),
    }
    if not args.no_cpu_baseline:
        import oracle
        t0 = time.perf_counter()
        for _ in range(3):
            oracle.adaln_modulation(oracle.adaln_code(e_b, basis_b), proj_b, bias_b)
        dt = (time.perf_counter() - t0) / 3
        line["cpu_baseline"] = {"value": by / dt / 1e9, "unit": "GB/s", "cores": len(os.sched_getaffinity(0)),
                                "kind": "oracle", "sample": "the whole call (8 timesteps, 42 blocks), 3 runs"}
    print(json.dumps(line))


# DRAM bytes (read + write) of one int8_scores_kernel launch on the workload
# above, from an ncu capture; valid only for the kernel source it was taken on.
ATTN_TRAFFIC = {"bytes": 1371803392, "source_sha256": "8d69c5a712786aec"}


def attn_traffic_valid():
    import hashlib
    path = os.path.join(ROOT, "nvfp4_quantized_linear_fh_b200", "csrc", "fh_int8.cu")
    with open(path, "rb") as f:
        digest = hashlib.sha256(f.read()).hexdigest()[:16]
    return ATTN_TRAFFIC["bytes"] is not None and digest == ATTN_TRAFFIC["source_sha256"]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    # 250 steps of ~0.4 ms: a ~0.1 s timed region, long enough for the clock
    # record to cover it and for the power limit to settle the clocks.
    ap.add_argument("--steps", type=int, default=250)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="fh", choices=["fh", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--M", type=int, default=WORKLOAD["M"],
                    help="token rows per GPU (profiling cases use fewer than the workload's 32768)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end measurement")
    ap.add_argument("--workload", default="qkv",
                    choices=["qkv", "tiny", "attn_proj", "ffn_pair", "block_sweep", "ffn", "attn", "adaln"],
                    help="qkv: the headline line (fused QKV layer), with the other four configurations in its "
                         "'configs' object; tiny, attn_proj, ffn_pair, block_sweep: one of those configurations "
                         "as a line of its own; ffn: the FFN block, fused vs unfused epilogue; attn: INT8 "
                         "query/key quantization and attention scores; adaln: AdaLN basis projection")
    ap.add_argument("--no-fused", action="store_true",
                    help="skip timing the quantization fused into the GEMM (fh_nvfp4_linear_fused_quant)")
    ap.add_argument("--no-configs", action="store_true",
                    help="headline line only (skip the other four configurations)")
    ap.add_argument("--quick", action="store_true",
                    help="calibrate on the input batches only (setup shortcut for profiling cases)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.workload == "ffn":
        bench_ffn(args)
        return
    if args.workload == "attn":
        bench_attn(args)
        return
    if args.workload == "adaln":
        bench_adaln(args)
        return
    if args.workload in ("tiny", "attn_proj", "ffn_pair", "block_sweep"):
        import torch
        torch.cuda.set_device(0)
        cfg = measure_configs(args, (args.workload,))[args.workload]
        print(json.dumps({"metric": METRIC, "workload": args.workload, "n_gpus": 1, "data": "synthetic", **cfg}))
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    pk = peaks()
    cfg = {"workload": f"fused QKV linear {args.M}x{WORKLOAD['K']}->{WORKLOAD['N']} (M x K -> N) per GPU",
           "M": args.M, "K": WORKLOAD["K"], "N": WORKLOAD["N"], "tokens_per_gpu": args.M,
           "parallelism": f"dp{world} (token rows per GPU, replicas)",
           "l2": "not flushed: each step's inputs and outputs exceed L2 (x 176 MB read, y 528 MB written)"}

    if args.impl == "reference":
        if rank != 0:
            return
        import synthetic as S
        layer = S.workloads()["qkv"][0]
        x_bits = S.activation_batches(layer, 0, 1)
        w_bits, b_bits = S.weights(layer), S.bias(layer)
        import oracle
        sg_a = oracle.scale_from_amax(oracle.amax(x_bits))
        sg_w = oracle.scale_from_amax(oracle.amax(w_bits))
        vals, secs = [], []
        for i in range(args.warmup + args.steps):
            v, dt, cores = cpu_baseline(x_bits, w_bits, b_bits, sg_a, sg_w, REF_ROWS)
            if i >= args.warmup:
                vals.append(v)
                secs.append(dt)
        value = statistics.median(vals)
        sample = (f"{REF_ROWS} token rows of the fused-QKV layer per step (quantize the rows, binary64 "
                  f"dequantized GEMM against weights quantized once beforehand)")
        print(json.dumps({"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS",
                          "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                          "ms_per_step": statistics.median(secs) * 1e3, "higher_is_better": True,
                          "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                          "config": cfg,
                          "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": cores, "kind": "oracle",
                                           "sample": sample},
                          "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0,
                                  "d2h_bytes_per_step": 0}}))
        return

    import torch
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    r = bench_fh(args, rank, world, local_rank)
    K_steps = args.steps
    value = r["flops"] * K_steps * world / r["t_step"] / 1e12
    gemm_mean = statistics.mean(r["t_gemm"])
    quant_mean = statistics.mean(r["t_quant"])
    achieved = r["flops"] / gemm_mean / 1e12
    fp4_sust = pk["bf16_sustained"] * FP4_OVER_BF16
    fp4_burst = pk["bf16"] * FP4_OVER_BF16
    # The denominator matches the regime of the timed region: a region under a
    # second runs before the power limit settles the clocks (the burst GEMM
    # figure); a longer one runs at the power-capped clocks (the sustained one).
    sustained = r["t_step"] >= 1.0
    fp4_peak = fp4_sust if sustained else fp4_burst
    quant_gbs = QUANT_BYTES_PER_ELEM * r["M"] * r["K"] / quant_mean / 1e9
    e2e_value = r["flops"] * r["e_steps"] * world / r["t_e2e"] / 1e12 if r["e_steps"] else None
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": K_steps,
        "warmup": args.warmup, "ms_per_step": r["t_step"] / K_steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4 (e2m1 x e4m3, fp32 accumulate, bf16 out)",
        "data": "synthetic (seeded; calibrated per-layer scale; random-init weights)", "config": cfg,
        "gpu_launches": 2 * K_steps,
        "roofline": {"kernel": "nvfp4_linear_kernel", "bound": "tensor", "achieved": achieved,
                     "peak": fp4_peak, "unit": "TFLOP/s", "frac": achieved / fp4_peak,
                     "peak_note": (f"{pk['source']} bf16 {'sustained' if sustained else 'burst'} "
                                   f"{pk['bf16_sustained'] if sustained else pk['bf16']} x 4 (nominal FP4/BF16); "
                                   f"timed region {r['t_step']:.3f} s "
                                   f"({'>=' if sustained else '<'} 1 s: {'sustained' if sustained else 'burst'})"),
                     "frac_of_burst_peak": achieved / fp4_burst,
                     "frac_of_sustained_peak": achieved / fp4_sust,
                     "traffic": gemm_traffic() if r["M"] == WORKLOAD["M"] else None,
                     "traffic_note": "bytes per launch, ncu dram__bytes_read.sum + dram__bytes_write.sum",
                     "algorithmic_bytes": gemm_bytes(r["M"], r["N"], r["K"])},
        "quantizer": {"kernel": "quantize_tiled_kernel", "bound": "hbm", "achieved": quant_gbs, "peak": pk["hbm_gbs"],
                      "unit": "GB/s", "frac": quant_gbs / pk["hbm_gbs"], "us": quant_mean * 1e6,
                      "traffic": quant_traffic() if r["M"] == WORKLOAD["M"] else None,
                      "algorithmic_bytes": QUANT_BYTES_PER_ELEM * r["M"] * r["K"]},
        "gemm_us": gemm_mean * 1e6, "clip_count": r["clips"],
        "e2e": {"value": e2e_value, "unit": "TFLOPS", "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"],
                "steps": r["e_steps"],
                "call": "fh_nvfp4_linear_host (pinned host x and y; upload, kernels and download overlapped over "
                        "4096-row chunks)"},
        "clocks": r["sampler"],
    }
    if r["t_fused"]:
        tf = statistics.mean(r["t_fused"])
        line["fused_quant"] = {"call": "fh_nvfp4_linear_fused_quant (quantization inside the GEMM kernel)",
                               "step_us": tf * 1e6, "tflops": r["flops"] / tf / 1e12,
                               "vs_two_calls": (r["t_step"] / K_steps) / tf, "steps": len(r["t_fused"]),
                               "output_identical_to_two_calls": True}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, dt, cores = cpu_baseline(r["x_bits"], r["w_bits"], r["b_bits"], r["sg_a"], r["sg_w"], CPU_SAMPLE_ROWS)
        line["cpu_baseline"] = {"value": v, "unit": "TFLOPS", "cores": cores, "kind": "oracle",
                                "sample": f"first {CPU_SAMPLE_ROWS} token rows of the same layer (quantize the rows, "
                                          f"binary64 dequantized GEMM; weights quantized beforehand), {dt:.1f} s"}
    if rank == 0:
        # The FP4 tensor rate measured with the library's own probe (no memory
        # traffic): the ceiling a block-scaled FP4 GEMM on this GPU can reach.
        r_mma, r_cp = fp4_tensor_rate(False) / 1e12, fp4_tensor_rate(True) / 1e12
        line["fp4_tensor_rate"] = {"mma_only": r_mma, "mma_with_scale_copies": r_cp, "unit": "TFLOP/s",
                                   "how": "fh_selftest_mma_rate: one CTA pair per SM pair, 60000 rounds of four "
                                          "256x256x64 kind::mxf4nvf4 MMAs from shared memory, best of 3"}
        line["roofline"]["frac_of_measured_fp4_rate"] = achieved / r_mma
    if rank == 0 and world == 1 and not args.no_configs and args.M == WORKLOAD["M"]:
        # The other four configurations, measured after the headline's timed region.
        line["configs"] = measure_configs(args)
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
