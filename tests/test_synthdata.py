"""The seeded input generators (shared by the tests and the benchmark; they
hold none of the method's arithmetic): determinism, shapes and the
distributions the workloads state.

* activations: channel i has standard deviation (i + 1)^-0.25 (variance
  (i + 1)^-0.5), four seeded channels scaled by 20;
* weights: N(0, std^2), rounded to the requested type;
* index sets: ascending, distinct, in range;
* the LLaMA layer's projection groups, with one rotation per distinct input.
"""
import numpy as np
import torch

import synthdata as sd


def test_seeds_are_deterministic_and_distinct():
    assert sd.seed_for(1, 2, 3) == 1_002_003
    a = sd.activations(2, 512, 77, torch.float32)
    b = sd.activations(2, 512, 77, torch.float32)
    c = sd.activations(2, 512, 78, torch.float32)
    assert torch.equal(a, b) and not torch.equal(a, c)
    assert torch.equal(sd.weights(64, 32, 0.02, 5), sd.weights(64, 32, 0.02, 5))


def test_activation_channel_scales_and_outliers():
    d, M = 256, 4000
    x = sd.activations(M, d, 123, torch.float32).double().numpy()
    std = x.std(axis=0)
    want = (np.arange(d) + 1.0) ** -0.25
    ratio = std / want
    outliers = np.nonzero(ratio > 10)[0]
    assert len(outliers) == 4
    np.testing.assert_allclose(ratio[outliers], 20.0, rtol=0.1)
    rest = np.delete(ratio, outliers)
    np.testing.assert_allclose(rest, 1.0, rtol=0.1)
    # bf16 rows are the same draws rounded
    xb = sd.activations(3, d, 5, torch.bfloat16)
    assert xb.dtype == torch.bfloat16
    assert torch.equal(xb, sd.activations(3, d, 5, torch.float32).to(torch.bfloat16))


def test_weights_scale_and_dtype():
    w = sd.weights(256, 512, 0.02, 9, torch.bfloat16)
    assert w.shape == (256, 512) and w.dtype == torch.bfloat16
    assert abs(float(w.double().std()) - 0.02) < 0.001
    w32 = sd.weights(256, 512, 1 / 16, 9, torch.float32)
    assert abs(float(w32.double().std()) - 1 / 16) < 0.002


def test_index_values_are_ascending_distinct_in_range():
    idx, val = sd.index_values(3, 1000, 400, 11)
    idx = idx.numpy()
    assert idx.shape == (3, 400) and val.shape == (3, 400)
    for row in idx:
        assert np.all(np.diff(row) > 0) and row[0] >= 0 and row[-1] < 1000


def test_llama_layer_groups():
    groups = sd.llama_layer(4096, 11008, 4096)
    assert [(g.name, g.d_in, g.d_out) for g in groups] == [
        ("qkv", 4096, 12288), ("o", 4096, 4096), ("gate_up", 4096, 22016), ("down", 11008, 4096)]
    # grouped-query attention: k and v narrower than q
    g70 = sd.llama_layer(8192, 28672, 1024)
    assert (g70[0].d_in, g70[0].d_out) == (8192, 8192 + 2 * 1024)
    # one rotation per distinct input: four distinct rotation ids
    assert len({g.q_id for g in groups}) == 4
