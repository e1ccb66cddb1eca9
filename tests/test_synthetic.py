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
