"""Device-resident synthetic LLaMA-shaped layers for tests and benchmarks.

Builds, for each projection group of a decoder layer (q|k|v, o, gate|up,
down), a seeded orthogonal rotation Q, a random weight W, its counter-rotated
form W_rot = Q^T W (computed by the library's own larosa_prepare_weights) and
a heavy-tailed activation x, all on one CUDA device.  Shapes only: no trained
weights are involved.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

import synthdata as sd

from .larosa import larosa_prepare_weights


@dataclass
class Group:
    """One projection group.  Qt is the rotation stored transposed (Q^T); W is
    the dense weight row-major [d_in, d_out], Wt the same in torch.nn.Linear
    layout [d_out, d_in] (used by the dense baseline); W_rot = Q^T W."""

    name: str
    d_in: int
    d_out: int
    K: int
    Qt: torch.Tensor
    W: torch.Tensor | None
    Wt: torch.Tensor | None
    W_rot: torch.Tensor
    x: torch.Tensor

    @property
    def rot_bytes(self) -> int:
        return self.Qt.numel() * self.Qt.element_size()

    def row_bytes(self, rows: int) -> int:
        return rows * self.d_out * self.W_rot.element_size()


@dataclass
class Layer:
    groups: list[Group] = field(default_factory=list)


def build_layer(hidden: int, ffn: int, kv: int, sparsity_pct: float, workload_id: int, layer: int,
                device: torch.device, M: int = 1, keep_dense: bool = True,
                w_std: float = 0.02, dtype: torch.dtype = torch.bfloat16) -> Layer:
    """One decoder layer's four projection groups, resident on ``device``."""
    out = Layer()
    for p in sd.llama_layer(hidden, ffn, kv):
        base = sd.seed_for(workload_id, layer, 10 * p.q_id)
        Qt = sd.orthogonal(p.d_in, base + 1, device=device).to(dtype).t().contiguous()
        W = sd.weights(p.d_in, p.d_out, w_std, base + 2, dtype, device=device)
        W_rot = larosa_prepare_weights(Qt, W)
        x = sd.activations(M, p.d_in, base + 3, dtype, device=device)
        K = sd.k_for_sparsity(p.d_in, sparsity_pct)
        Wt = W.t().contiguous() if keep_dense else None
        out.groups.append(Group(p.name, p.d_in, p.d_out, K, Qt, W if keep_dense else None, Wt,
                                W_rot, x))
    torch.cuda.synchronize(device)
    return out
