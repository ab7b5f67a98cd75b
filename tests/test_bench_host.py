"""Host-side logic of the benchmark, on the CPU.

* The algorithmic byte count of one token through a LLaMA2-7B-shaped layer
  at 40 % sparsity: kept rows K * d_out * 2 (bf16), the rotation d^2 * 2,
  and the activations.  The kept-row and rotation totals are fixed by the
  shapes alone (242.88 MB of rows and 343.0 MB of rotations, 585.9 MB in
  all before the activations), so a dropped term or a wrong K shows up here.
* The perf-only layers of the larger workloads: their rotations are signed
  row permutations of one Haar rotation per width, which must still be
  orthogonal, distinct per layer and group, and of the right shapes.
* The reference arm (the fp64 oracle on the host cores) prints exactly one
  JSON line with the benchmark's keys.
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import bench
import synthdata as sd


class _G:
    def __init__(self, d_in, d_out):
        self.d_in, self.d_out = d_in, d_out


def test_path_bytes_llama2_7b_layer():
    groups = [_G(p.d_in, p.d_out) for p in sd.llama_layer(4096, 11008, 4096)]
    Ks = [sd.k_for_sparsity(g.d_in, 40.0) for g in groups]
    assert Ks == [2458, 2458, 2458, 6605]
    parts = [bench.path_bytes(g, K) for g, K in zip(groups, Ks)]
    rows = sum(p["rows"] for p in parts)
    q = sum(p["q"] for p in parts)
    # kept rows: 2458 * (12288 + 4096 + 22016) * 2 + 6605 * 4096 * 2
    assert rows == 2458 * (12288 + 4096 + 22016) * 2 + 6605 * 4096 * 2
    assert rows == pytest.approx(242.88e6, rel=1e-4)
    assert q == 3 * 4096 * 4096 * 2 + 11008 * 11008 * 2
    assert rows + q == pytest.approx(585.9e6, rel=1e-4)
    # the activations are a small remainder: x, x_rot, the kept list, y
    total = sum(p["total"] for p in parts)
    act = sum(p["act"] for p in parts)
    assert act == sum(g.d_in * 6 + K * 8 + g.d_out * 4 for g, K in zip(groups, Ks))
    assert total == rows + q + act and act < 1e-3 * total
    # without the rotation only Q's bytes go
    assert sum(bench.path_bytes(g, K, rotate=False)["total"] for g, K in zip(groups, Ks)) == total - q


def test_path_bytes_dense_equivalent_at_zero_sparsity():
    g = _G(256, 512)
    b = bench.path_bytes(g, 256, rotate=False)
    assert b["rows"] == 256 * 512 * 2


def test_perf_layers_rotations_are_orthogonal_and_distinct():
    layers = bench.perf_layers(torch, sd, 64, 96, 32, 2, 7, 3, "cpu")
    assert len(layers) == 2
    names = [g.name for g in layers[0]]
    assert names == ["qkv", "o", "gate_up", "down"]
    shapes = [(g.d_in, g.d_out) for g in layers[0]]
    assert shapes == [(64, 64 + 2 * 32), (64, 64), (64, 192), (96, 64)]
    seen = []
    for gs in layers:
        for g in gs:
            assert g.Qt.shape == (g.d_in, g.d_in) and g.Qt.dtype == torch.bfloat16
            assert g.W_rot.shape == (g.d_in, g.d_out) and g.W_rot.dtype == torch.bfloat16
            assert g.x.shape == (3, g.d_in)
            q = g.Qt.double()
            # orthogonal up to the bf16 rounding of its entries (2^-9 relative)
            err = np.abs((q @ q.t()).numpy() - np.eye(g.d_in)).max()
            assert err < 0.02, err
            seen.append(q)
    # every layer and group has its own rotation
    for i in range(len(seen)):
        for j in range(i + 1, len(seen)):
            if seen[i].shape == seen[j].shape:
                assert not torch.equal(seen[i], seen[j])


def test_perf_layers_weight_scale():
    layers = bench.perf_layers(torch, sd, 128, 256, 128, 1, 8, 1, "cpu")
    w = torch.cat([g.W_rot.double().flatten() for g in layers[0]])
    assert float(w.std()) == pytest.approx(0.02, rel=0.05)
    assert abs(float(w.mean())) < 1e-3


def test_reference_arm_prints_one_json_line_with_the_contract_keys():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3"], capture_output=True, text=True, timeout=600, check=True).stdout
    lines = [ln for ln in out.splitlines() if ln.strip()]
    assert len(lines) == 1, lines
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["dtype"] == "f64" and d["data"] == "synthetic"
    assert d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 3 and d["higher_is_better"] is True
    assert d["unit"] == "tokens/s" and d["value"] > 0 and d["ms_per_step"] > 0
    assert "llama2-7b-layer" in d["config"]["workload"]
    cpu = d["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["cores"] >= 1 and cpu["value"] == d["value"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
