"""A small, fixed workload for kernel profilers (ncu): one LLaMA2-7B-shaped
projection group, batch 1, run a few times through each decode entry point.

    python -m activation_sparsity_b200.profile_case [--group gate_up] [--iters 3]
                                                    [--sparsity 40]

Each iteration launches, in this order: the fused call (rotation kernel, then
the select-and-gather kernel), the sparse linear on a fixed kept list (list
gather kernel) and the dense baseline (rotation kernel on W in nn.Linear
layout).  The group's tensors take 0.2-0.5 GB of device memory, more than the
126 MB L2, and ncu flushes the caches before every replayed launch, so DRAM
counters describe cold-cache launches.  Prints "ok" and exits 0 on success.
"""
from __future__ import annotations

import argparse
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synthdata as sd  # noqa: E402

from . import larosa as L  # noqa: E402

GROUPS = {p.name: p for p in sd.llama_layer(4096, 11008, 4096)}


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__,
                                 formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--group", choices=sorted(GROUPS), default="gate_up")
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--sparsity", type=float, default=40.0)
    a = ap.parse_args(argv)
    if not torch.cuda.is_available():
        raise SystemExit("profile_case: no CUDA device (the library has no CPU path)")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    p = GROUPS[a.group]
    base = sd.seed_for(1, 0, 10 * p.q_id)
    Qt = sd.orthogonal(p.d_in, base + 1, device=dev).to(torch.bfloat16).t().contiguous()
    W = sd.weights(p.d_in, p.d_out, 0.02, base + 2, torch.bfloat16, device=dev)
    W_rot = L.larosa_prepare_weights(Qt, W)
    Wt = W.t().contiguous()
    del W
    x = sd.activations(1, p.d_in, base + 3, torch.bfloat16, device=dev)
    K = sd.k_for_sparsity(p.d_in, a.sparsity)
    ws = L.Workspace(dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    y = torch.empty((1, p.d_out), dtype=torch.float32, device=dev)
    x_rot = L.larosa_rotate(x, Qt)
    idx, val = L.larosa_topk(x_rot, K, dev_status=st)
    for _ in range(a.iters):
        L.larosa_rotate_topk_linear(x, Qt, W_rot, K, y=y, ws=ws, dev_status=st)
        L.larosa_sparse_linear(idx, val, W_rot, y=y, ws=ws, dev_status=st)
        L.larosa_dense_linear(x, Wt, y=y)
    torch.cuda.synchronize(dev)
    if L.larosa_check(st, device=dev) != 0:
        raise SystemExit("profile_case: the library reported a device status")
    print(f"ok: {a.group} d_in={p.d_in} d_out={p.d_out} K={K} iters={a.iters}")
    return 0


if __name__ == "__main__":
    sys.exit(main())
