"""The seeded input generators: determinism, BF16 rounding, recipe structure."""
import numpy as np
import torch

import synthetic as S


def test_bf16_rounding_matches_torch_on_float32_inputs():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-6, 6, 20000),
                        [0.0, -0.0, 1.0, -2.5, 1.00390625, 1.01171875, 65504.0]]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(S.to_bf16_bits(x.astype(np.float64)), ref)


def test_streams_are_counter_based_and_deterministic():
    a = S.normal(123, 0, 1001)
    b = np.concatenate([S.normal(123, 0, 400), S.normal(123, 400, 601)])
    np.testing.assert_array_equal(a, b)
    assert abs(a.mean()) < 0.1 and abs(a.std() - 1) < 0.1
    u = S.uniform(5, 0, 100000)
    assert u.min() > 0 and u.max() < 1


def test_tiny_recipe_structure():
    layer = S.workloads()["tiny"][0]
    x = S.activations(layer)
    assert x.shape == (128, 256)
    v = S.bf16_to_f32(x).reshape(-1)
    pos = S.outlier_positions(layer, 0)
    assert pos.size == 33
    np.testing.assert_array_equal(np.abs(v[pos]), 1096.0)
    assert np.abs(np.delete(v, pos)).max() < S.CLIP_LIMIT
    np.testing.assert_array_equal(S.activation_batches(layer, 0, 1), x)


def test_eval_input_is_prefix_of_calibration_stream():
    layer = S.workloads()["attn_proj"][0]
    two = S.activation_batches(layer, 0, 2)
    np.testing.assert_array_equal(S.activation_batches(layer, 1, 1), two[64:])
    v = S.bf16_to_f32(two)
    assert v.shape == (128, 2688)
    assert np.abs(v).max() == 1096.0           # one outlier of each batch is exactly 137 L


def test_weights_and_bias_distributions():
    layer = S.workloads()["tiny"][0]
    w = S.bf16_to_f32(S.weights(layer))
    b = S.bf16_to_f32(S.bias(layer))
    assert w.shape == (256, 256) and b.shape == (256,)
    assert abs(w.std() - 0.02) < 0.002 and abs(b.std() - 0.01) < 0.003


def test_f16_rounding_matches_torch():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-8, 5, 20000),
                        [0.0, -0.0, 1.0, 65504.0, 65520.0, 2.0 ** -24, 2.0 ** -25, 1.0 + 2.0 ** -11]])
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    with np.errstate(over="ignore"):                            # 65520 rounds to +inf on purpose
        np.testing.assert_array_equal(S.to_f16_bits(x.astype(np.float32)), ref)


def test_attention_qk_structure():
    """Per-(head, channel) spreads, about one outlier channel in 32 at 8x, every
    tenth token at 4x; queries and keys differ, the same call repeats."""
    h, t, d = 4, 400, 256
    q = S.attention_qk(h, t, d, "q")
    assert q.shape == (h, t, d) and q.dtype == np.uint16
    np.testing.assert_array_equal(q, S.attention_qk(h, t, d, "q"))
    assert not np.array_equal(q, S.attention_qk(h, t, d, "k"))
    v = S.bf16_to_f32(q).astype(np.float64)
    body = np.delete(v, np.arange(0, t, 10), axis=1)
    ch_std = body.std(axis=1)                                   # [h, d]
    loud = ch_std > 8.0 * np.median(ch_std)
    assert 0 < loud.sum() < h * d // 8
    tenth = v[:, ::10, :]
    ratio = np.abs(tenth).mean() / np.abs(body).mean()
    assert 3.0 < ratio < 5.0


def test_adaln_inputs_shapes_and_spreads():
    e, basis, proj, bias = S.adaln_inputs(3, 500, 2688, 16, S.SAMPLER_TIMESTEPS, seed=2)
    assert e.shape == (8, 2688) and basis.shape == (16, 2688)
    assert proj.shape == (3, 500, 16) and bias.shape == (3, 500)
    f16 = lambda b: b.view(np.float16).astype(np.float64)  # noqa: E731
    assert abs(S.bf16_to_f32(e).std() - 1.0) < 0.05
    assert np.allclose(np.linalg.norm(f16(basis), axis=1), 1.0, atol=0.05)
    assert abs(f16(proj).std() - 0.05) < 0.005 and abs(f16(bias).std() - 0.01) < 0.002
    # One seeded embedding per timestep: the same timestep gives the same row.
    e2, *_ = S.adaln_inputs(1, 1, 2688, 16, (125, 999), seed=2)
    np.testing.assert_array_equal(e2, e[[7, 0]])
    e0, *_ = S.adaln_inputs(1, 1, 64, 16, ())
    assert e0.shape == (0, 64)


def test_torch_recipes_match_numpy_recipes_on_cpu():
    """The torch restatement of the generator (used on the GPU for the full-size
    workloads) gives the numpy recipe's BF16 bits: streams at odd offsets, the
    log-normal channel spread, plain bodies, weights and biases."""
    import torch
    u = S.u64(12345678901234567890, 3, 7)
    assert np.array_equal(u, S.u64_t(12345678901234567890, 3, 7, "cpu").numpy().view(np.uint64))
    assert np.array_equal(S.normal(77, 5, 11), S.normal_t(77, 5, 11, "cpu").numpy())
    sw = S.workloads()["block_sweep"]
    for layer in (sw[0], sw[3]):                       # qkv-like (log-normal channels) and down (plain)
        small = S.Layer(layer.name, 256, layer.K, 512, layer.batch, 8,
                        channel_lognormal=layer.channel_lognormal, key=layer.key)
        want = S.activation_batches(small, 2, 3)
        got = S.activation_batches_t(small, 2, 3, "cpu").numpy().view(np.uint16)
        assert np.array_equal(want, got)
        assert np.array_equal(S.weights(small), S.weights_t(small, "cpu").numpy().view(np.uint16))
        assert np.array_equal(S.bias(small), S.bias_t(small, "cpu").numpy().view(np.uint16))
    x = np.array([1.0, -1.00390625, 1.001953125, 1.005859375, 3.0e38, -0.0, 65504.5, -7.99])
    assert np.array_equal(S.to_bf16_bits(x), S.to_bf16_bits_t(torch.from_numpy(x)).numpy().view(np.uint16))


def test_torch_recipes_redraw_like_numpy():
    """With a truncation bound of 1.5 (a third of the draws redrawn, some more
    than once) the torch path redraws exactly as the numpy path does."""
    layer = S.workloads()["block_sweep"][3]
    small = S.Layer(layer.name, 64, 64, 64, 8, 3, key=layer.key)
    want = S.activation_batches(small, 0, 3, bound=1.5)
    got = S.activation_batches_t(small, 0, 3, "cpu", chunk=2, bound=1.5).numpy().view(np.uint16)
    assert np.array_equal(want, got)
    assert (np.abs(S.bf16_to_f32(want)) <= 1.5).all()       # < 1.5 before the BF16 rounding


def test_torch_recipes_inject_outliers_like_numpy():
    """Both outlier modes: fixed +-137 L (tiny workload) and L * U[1, 137] with
    one exactly 137 L per batch (attention projection), at the same positions,
    signs and magnitudes as the numpy recipe."""
    tiny = S.workloads()["tiny"][0]
    assert np.array_equal(S.activation_batches(tiny, 3, 2), S.activation_batches_t(tiny, 3, 2, "cpu").numpy().view(np.uint16))
    ap = S.workloads()["attn_proj"][0]
    small = S.Layer(ap.name, 128, 512, 64, ap.batch, 4, ap.outlier_rate * 8, ap.outlier_mode, key=ap.key)
    assert small.outliers_per_batch() > 1
    want = S.activation_batches(small, 1, 2)
    assert np.array_equal(want, S.activation_batches_t(small, 1, 2, "cpu").numpy().view(np.uint16))
