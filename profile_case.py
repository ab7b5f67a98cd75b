"""A small, fixed workload for kernel profilers (ncu): one LLaMA2-7B-shaped
projection group, run a few times through each decode entry point.

    python profile_case.py [--group gate_up|all] [--iters 3] [--sparsity 40]
                           [--fused-only] [--tokens M]

For each group (``all``: q|k|v, o, gate|up, down in that order) each
iteration launches, for one token: the fused call (one fused_kernel), the
Top-K of a pre-rotated input (topk_kernel), the sparse linear on a fixed kept
list (gather_kernel), the dense baseline (rowdot_kernel on W in nn.Linear
layout) and the Top-K + sparse linear of the pre-rotated input in one call
(topk_kernel, gather_kernel); ``--fused-only`` launches only the fused call.  With ``--tokens M``
(2 to 16) each iteration runs M tokens through the same entry points: the
rotation, the Top-K, the multi-token sparse linear and the fused call (for
8 to 16 tokens the tcgen05 kernels).  One group takes 0.2-0.5 GB of device
memory, more than the 126 MB L2, and ncu flushes the caches before every
replayed launch, so DRAM counters describe cold-cache launches.  Prints "ok"
and exits 0 on success.
"""
from __future__ import annotations

import argparse
import os
import sys

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synthdata as sd  # noqa: E402
from activation_sparsity_b200 import larosa as L  # noqa: E402

GROUPS = {p.name: p for p in sd.llama_layer(4096, 11008, 4096)}


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__,
                                 formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--group", choices=sorted(GROUPS) + ["all"], default="gate_up")
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--sparsity", type=float, default=40.0)
    ap.add_argument("--fused-only", action="store_true")
    ap.add_argument("--tokens", type=int, default=1)
    a = ap.parse_args(argv)
    if not 1 <= a.tokens <= 16:
        ap.error("--tokens must be 1 to 16")
    if not torch.cuda.is_available():
        raise SystemExit("profile_case: no CUDA device (the library has no CPU path)")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    names = [p.name for p in sd.llama_layer(4096, 11008, 4096)] if a.group == "all" else [a.group]
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = L.Workspace(dev)
    cases = []
    for name in names:
        p = GROUPS[name]
        base = sd.seed_for(1, 0, 10 * p.q_id)
        Qt = sd.orthogonal(p.d_in, base + 1, device=dev).to(torch.bfloat16).t().contiguous()
        W = sd.weights(p.d_in, p.d_out, 0.02, base + 2, torch.bfloat16, device=dev)
        W_rot = L.larosa_prepare_weights(Qt, W)
        Wt = None if a.fused_only else W.t().contiguous()
        del W
        M = a.tokens
        x = sd.activations(M, p.d_in, base + 3, torch.bfloat16, device=dev)
        K = sd.k_for_sparsity(p.d_in, a.sparsity)
        y = torch.empty((M, p.d_out), dtype=torch.float32, device=dev)
        x_rot = idx = val = None
        if not a.fused_only:
            x_rot = L.larosa_rotate(x, Qt)
            idx, val = L.larosa_topk(x_rot, K, dev_status=st)
        cases.append((p, Qt, W_rot, Wt, x, K, y, x_rot, idx, val))
    for _ in range(a.iters):
        for p, Qt, W_rot, Wt, x, K, y, x_rot, idx, val in cases:
            L.larosa_rotate_topk_linear(x, Qt, W_rot, K, y=y, ws=ws, dev_status=st)
            if not a.fused_only:
                if a.tokens > 1:
                    L.larosa_rotate(x, Qt, x_rot=x_rot)
                L.larosa_topk(x_rot, K, idx=idx, val=val, dev_status=st)
                L.larosa_sparse_linear(idx, val, W_rot, y=y, ws=ws, dev_status=st)
                L.larosa_dense_linear(x, Wt, y=y)
                L.larosa_topk_linear(x_rot, W_rot, K, y=y, ws=ws, dev_status=st)
    torch.cuda.synchronize(dev)
    if L.larosa_check(st, device=dev) != 0:
        raise SystemExit("profile_case: the library reported a device status")
    print(f"ok: groups {','.join(names)} tokens {a.tokens} sparsity {a.sparsity}% iters {a.iters}")
    return 0


if __name__ == "__main__":
    sys.exit(main())
