"""Seeded synthetic inputs for the rotated-sparse linear path.

This module produces the *inputs* both the CUDA library and the fp64 oracle
consume: activations, weights, orthogonal rotations and the per-projection
shapes of the LLaMA2 families.  It holds none of the method's arithmetic (no
rotation of activations, no Top-K, no counter-rotation of weights): the
random numbers it draws are handed to both sides as plain tensors.

Recipes (stated once here, restated in the design notes):

* Orthogonal Q: the Q factor of a QR factorisation of a seeded N(0, 1) square
  matrix, with column signs fixed so that diag(R) > 0 (a Haar-distributed
  rotation).  The LaRoSA pages leave the choice of Q open ("random
  initialisation or learned", La RoSA summary, "关键设计" paragraph); a seeded
  random rotation stands in because trained models are not available.
* Activations x: per-channel standard deviation (i+1)^-0.25 (variance
  (i+1)^-0.5) plus four seeded distinct outlier channels multiplied by 20,
  the heavy-tailed channel structure of LLM hidden states.
* Weights W ~ N(0, std^2), std 0.02 for the LLaMA-shaped workloads and 1/16
  for the 256-wide single projection.

Seeds follow ``seed = 1_000_000 * workload + 1000 * layer + tensor_id``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

__all__ = [
    "seed_for",
    "k_for_sparsity",
    "orthogonal",
    "activations",
    "weights",
    "index_values",
    "Projection",
    "llama_layer",
    "WORKLOADS",
]


def seed_for(workload: int, layer: int, tensor_id: int) -> int:
    """Deterministic seed of one tensor of one layer of one workload."""
    return 1_000_000 * workload + 1000 * layer + tensor_id


def k_for_sparsity(d: int, sparsity_pct: float) -> int:
    """Number of kept entries K for sparsity ``sparsity_pct`` percent of ``d``.

    K = d - floor(s * d / 100), so the achieved sparsity never exceeds s.
    (40 % of 256 keeps 154; 40 % of 4096 keeps 2458; 40 % of 11008 keeps 6605.)
    """
    if not (0.0 <= sparsity_pct <= 100.0):
        raise ValueError("sparsity must lie in [0, 100] percent")
    dropped = math.floor(sparsity_pct * d / 100.0 + 1e-9)
    return d - dropped


def orthogonal(d: int, seed: int, device: str | torch.device = "cpu") -> torch.Tensor:
    """Seeded Haar-random orthogonal d x d matrix.

    On the CPU the factorisation runs in fp64 with numpy (PCG64 stream) and the
    result is an fp64 tensor; on a CUDA device a torch generator seeded with
    ``seed`` draws the Gaussian matrix and the factorisation runs in fp32
    (used for the large perf-only rotations, where fp64 CPU QR would take
    minutes).  Only the rotation's values matter to the path, not how they
    were obtained.
    """
    device = torch.device(device)
    if device.type == "cpu":
        rng = np.random.default_rng(seed)
        g = rng.standard_normal((d, d))
        q, r = np.linalg.qr(g)
        q = q * np.sign(np.where(np.diag(r) == 0, 1.0, np.diag(r)))[None, :]
        return torch.from_numpy(np.ascontiguousarray(q))
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    g = torch.randn((d, d), generator=gen, device=device, dtype=torch.float32)
    q, r = torch.linalg.qr(g)
    s = torch.sign(torch.diagonal(r))
    s[s == 0] = 1.0
    return (q * s[None, :]).contiguous()


def _channel_std(d: int, seed: int) -> np.ndarray:
    std = (np.arange(d, dtype=np.float64) + 1.0) ** -0.25
    rng = np.random.default_rng(seed + 7)
    n_out = min(4, d)
    outliers = rng.choice(d, size=n_out, replace=False)
    std[outliers] *= 20.0
    return std


def activations(M: int, d: int, seed: int, dtype: torch.dtype = torch.bfloat16,
                device: str | torch.device = "cpu") -> torch.Tensor:
    """M heavy-tailed activation rows of width d, rounded to ``dtype``.

    Draws are made on the CPU in fp64 (PCG64) and cast, so the values do not
    depend on the device they are placed on.
    """
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((M, d))
    x = z * _channel_std(d, seed)[None, :]
    return torch.from_numpy(x).to(dtype).to(device)


def weights(d_in: int, d_out: int, std: float, seed: int,
            dtype: torch.dtype = torch.bfloat16,
            device: str | torch.device = "cpu") -> torch.Tensor:
    """Row-major [d_in x d_out] weight ~ N(0, std^2), rounded to ``dtype``.

    Small matrices are drawn on the CPU (PCG64, device independent); matrices
    above 2^24 entries are drawn with a seeded torch generator on ``device``
    to keep perf-only setup fast.
    """
    device = torch.device(device)
    if d_in * d_out <= (1 << 24) or device.type == "cpu":
        rng = np.random.default_rng(seed)
        w = rng.standard_normal((d_in, d_out), dtype=np.float32) * np.float32(std)
        return torch.from_numpy(w).to(dtype).to(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    w = torch.randn((d_in, d_out), generator=gen, device=device, dtype=torch.float32)
    return (w * std).to(dtype)


def index_values(M: int, d: int, K: int, seed: int) -> tuple[torch.Tensor, torch.Tensor]:
    """Seeded ascending index sets (M x K, int32) and fp32 values (M x K).

    Used to drive the sparse linear on its own, independent of any selection.
    """
    rng = np.random.default_rng(seed)
    idx = np.empty((M, K), dtype=np.int32)
    for m in range(M):
        idx[m] = np.sort(rng.choice(d, size=K, replace=False)).astype(np.int32)
    val = rng.standard_normal((M, K)).astype(np.float32)
    return torch.from_numpy(idx), torch.from_numpy(val)


@dataclass(frozen=True)
class Projection:
    """One projection group: the linears that share one input activation."""

    name: str
    d_in: int
    d_out: int
    q_id: int          # which rotation of the layer it reads (shared inputs share one)


def llama_layer(hidden: int, ffn: int, kv_out: int | None = None) -> list[Projection]:
    """The four projection groups of a LLaMA decoder layer, in execution order.

    q|k|v read the attention input, o reads the attention output, gate|up read
    the MLP input and down reads the MLP hidden state: one rotation per
    distinct input (La RoSA summary, "技术框架": one orthogonal rotation per
    layer input).
    """
    kv = hidden if kv_out is None else kv_out
    return [
        Projection("qkv", hidden, hidden + 2 * kv, 0),
        Projection("o", hidden, hidden, 1),
        Projection("gate_up", hidden, 2 * ffn, 2),
        Projection("down", ffn, hidden, 3),
    ]


# Named workloads (shapes only; no trained weights are involved).
WORKLOADS = {
    "tiny-256x512": dict(kind="single", d_in=256, d_out=512, M=1, dtype="fp32", w_std=1.0 / 16.0),
    "llama2-7b-layer": dict(kind="layer", hidden=4096, ffn=11008, kv=4096, layers=1, w_std=0.02),
    "llama2-7b-stack": dict(kind="layer", hidden=4096, ffn=11008, kv=4096, layers=32, w_std=0.02),
    "llama2-13b-layer": dict(kind="layer", hidden=5120, ffn=13824, kv=5120, layers=1, w_std=0.02),
    "llama2-70b-slice": dict(kind="layer", hidden=8192, ffn=28672, kv=1024, layers=8, w_std=0.02),
}


ADVERSARIAL_KINDS = ("gaussian", "heavy", "small_ints", "equal_magnitude", "ulp_neighbours",
                     "subnormal", "zeros")


def adversarial_rows(kind: str, M: int, d: int, seed: int) -> torch.Tensor:
    """fp32 [M x d] rows that stress a magnitude selection.

    gaussian         N(0, 1)
    heavy            the heavy-tailed activation recipe, in fp32
    small_ints       integers in [-3, 3] (many equal magnitudes, +0 and -0)
    equal_magnitude  +-1.5 with random signs (every magnitude ties)
    ulp_neighbours   1.0 and its next fp32 neighbours, random signs
    subnormal        fp32 subnormals and zeros
    zeros            +0 and -0 only
    """
    rng = np.random.default_rng(seed)
    if kind == "gaussian":
        a = rng.standard_normal((M, d))
    elif kind == "heavy":
        a = rng.standard_normal((M, d)) * _channel_std(d, seed)[None, :]
    elif kind == "small_ints":
        a = rng.integers(-3, 4, size=(M, d)).astype(np.float64)
        a[rng.random((M, d)) < 0.1] = -0.0
    elif kind == "equal_magnitude":
        a = np.where(rng.random((M, d)) < 0.5, -1.5, 1.5)
    elif kind == "ulp_neighbours":
        one = np.float32(1.0)
        vals = np.array([np.nextafter(one, np.float32(0)), one, np.nextafter(one, np.float32(2))],
                        dtype=np.float32)
        a = vals[rng.integers(0, 3, size=(M, d))].astype(np.float64)
        a *= np.where(rng.random((M, d)) < 0.5, -1.0, 1.0)
    elif kind == "subnormal":
        a = rng.integers(-40, 41, size=(M, d)).astype(np.float64) * 2.0 ** -149
    elif kind == "zeros":
        a = np.where(rng.random((M, d)) < 0.5, -0.0, 0.0)
    else:
        raise ValueError(kind)
    return torch.from_numpy(a.astype(np.float32))
