"""The multi-GPU host path with two gloo ranks on CPU: row sharding,
calibration amax all-reduce, clip-count sum and max-over-ranks timing.  The
per-rank arithmetic is the oracle's (no GPU here); the point is that sharded
calibration and quantization reproduce the unsharded results exactly, and that
the INT8 attention scores (by head) and the AdaLN projection (by timestep and
by block) split into replicas whose shares reassemble the unsharded result."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    import oracle
    import synthetic as S
    from nvfp4_quantized_linear_fh_b200 import dist as fhd
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        layer = S.workloads()["tiny"][0]
        # Calibration batches are split between ranks; the global amax is their MAX.
        mine = [b for b in range(layer.n_calib) if b % world == rank]
        local = max(oracle.amax(S.activation_batches(layer, b, 1)) for b in mine)
        amax = fhd.global_amax(torch.tensor([local], dtype=torch.float32))
        sg = oracle.scale_from_amax(float(amax.item()))
        # Each rank quantizes its rows of the input.
        x = S.activations(layer)
        r0, r1 = fhd.shard_rows(layer.M, world, rank, align=32)
        codes, scales, clip = oracle.quantize(x[r0:r1], sg)
        clips = fhd.total_clips(torch.tensor([clip], dtype=torch.int64))
        t = fhd.max_over_ranks([0.5 + rank, 3.0 - rank])
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), codes=codes, scales=scales, r=np.array([r0, r1]),
                 sg=np.array([sg]), clips=np.array([int(clips.item())]), t=np.array(t))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_sharded_calibration_and_quantization_match_unsharded(tmp_path, world):
    import oracle
    import synthetic as S
    mp.spawn(_worker, args=(world, free_port(), str(tmp_path)), nprocs=world, join=True)
    layer = S.workloads()["tiny"][0]
    sg_ref = oracle.scale_from_amax(oracle.amax(S.activation_batches(layer, 0, layer.n_calib)))
    x = S.activations(layer)
    codes_ref, scales_ref, clip_ref = oracle.quantize(x, sg_ref)
    parts = [np.load(tmp_path / f"rank{r}.npz") for r in range(world)]
    assert all(p["sg"][0] == sg_ref for p in parts)
    rows = [tuple(p["r"]) for p in parts]
    assert rows[0][0] == 0 and rows[-1][1] == layer.M
    assert all(rows[i][1] == rows[i + 1][0] for i in range(world - 1))
    np.testing.assert_array_equal(np.concatenate([p["codes"] for p in parts]), codes_ref)
    np.testing.assert_array_equal(np.concatenate([p["scales"] for p in parts]), scales_ref)
    assert all(p["clips"][0] == clip_ref for p in parts)
    assert all(list(p["t"]) == [0.5 + world - 1, 3.0] for p in parts)


def test_shard_rows_partitions():
    from nvfp4_quantized_linear_fh_b200.dist import shard_rows
    for M in [0, 1, 127, 128, 1000, 32768, 49152]:
        for world in [1, 2, 3, 8]:
            for align in [1, 128, 256]:
                spans = [shard_rows(M, world, r, align) for r in range(world)]
                assert spans[0][0] == 0 and spans[-1][1] == M
                assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
                units = [-(-(b - a) // align) for a, b in spans]
                assert max(units) - min(units) <= 1
                assert all(a % align == 0 for a, b in spans if b > a)
    with pytest.raises(ValueError):
        shard_rows(10, 2, 2)


def _replica_worker(rank, world, port, out_dir):
    """The secondary workloads as replicas: attention scores split by head, AdaLN
    codes by timestep and modulations by block, each rank computing its share
    with no exchange in the data path (only the barrier the bench takes)."""
    import sys
    sys.path.insert(0, ROOT)
    import oracle
    import synthetic as S
    from nvfp4_quantized_linear_fh_b200 import dist as fhd
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        H, T, d = 5, 40, 32
        q = S.attention_qk(H, T, d, "q", seed=7)
        k = S.attention_qk(H, T, d, "k", seed=7)
        h0, h1 = fhd.shard_rows(H, world, rank)
        q8, qs = oracle.quantize_int8_rows(q[h0:h1].reshape(-1, d))
        k8, ks = oracle.quantize_int8_rows(k[h0:h1].reshape(-1, d))
        n = h1 - h0
        s = oracle.int8_scores(q8.reshape(n, T, d), qs.reshape(n, T), k8.reshape(n, T, d), ks.reshape(n, T),
                               d ** -0.5)
        e, basis, proj, bias = S.adaln_inputs(3, 24, 64, 16, S.SAMPLER_TIMESTEPS, seed=5)
        t0, t1 = fhd.shard_rows(e.shape[0], world, rank)
        code = oracle.adaln_code(e[t0:t1], basis)
        l0, l1 = fhd.shard_rows(proj.shape[0], world, rank)
        mod = oracle.adaln_modulation(oracle.adaln_code(e, basis), proj[l0:l1], bias[l0:l1])
        dist.barrier()
        np.savez(os.path.join(out_dir, f"replica{rank}.npz"), s=s, code=code, mod=mod)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_secondary_workloads_shard_without_exchange(tmp_path, world):
    import oracle
    import synthetic as S
    mp.spawn(_replica_worker, args=(world, free_port(), str(tmp_path)), nprocs=world, join=True)
    parts = [np.load(tmp_path / f"replica{r}.npz") for r in range(world)]
    H, T, d = 5, 40, 32
    q8, qs = oracle.quantize_int8_rows(S.attention_qk(H, T, d, "q", seed=7).reshape(-1, d))
    k8, ks = oracle.quantize_int8_rows(S.attention_qk(H, T, d, "k", seed=7).reshape(-1, d))
    s_ref = oracle.int8_scores(q8.reshape(H, T, d), qs.reshape(H, T), k8.reshape(H, T, d), ks.reshape(H, T),
                               d ** -0.5)
    np.testing.assert_array_equal(np.concatenate([p["s"] for p in parts]), s_ref)
    e, basis, proj, bias = S.adaln_inputs(3, 24, 64, 16, S.SAMPLER_TIMESTEPS, seed=5)
    code_ref = oracle.adaln_code(e, basis)
    np.testing.assert_array_equal(np.concatenate([p["code"] for p in parts]), code_ref)
    np.testing.assert_array_equal(np.concatenate([p["mod"] for p in parts]),
                                  oracle.adaln_modulation(code_ref, proj, bias))
