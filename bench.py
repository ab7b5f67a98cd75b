#!/usr/bin/env python
"""Benchmark of the LaRoSA rotated-sparse linear path on one node.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl larosa|reference]
                    [--sparsity 40]

A step is one decode token through the whole path of one LLaMA2-7B-shaped
decoder layer: for each of its four projection groups (q|k|v 4096x12288,
o 4096x4096, gate|up 4096x22016, down 11008x4096) rotate the input by the
group's own orthogonal Q, keep the exact Top-K (40 % sparsity: K = 2458 of
4096, 6605 of 11008) and multiply by the counter-rotated weight, reading only
the kept rows.  Inputs are seeded and synthetic; weights are random of the
right shapes.

Timed with CUDA events on the launching stream after W warm-up steps, the K
steps replayed from a CUDA graph of one step; the working set (586 MB of
rotations and kept weight rows per step) exceeds the 126 MB L2, so no flush is
needed.  N > 1 runs N independent replicas (one process per GPU, no data-path
collective); the reported time is the maximum over ranks.

Rank 0 prints one JSON line.  Besides the headline it carries, from the same
run: the roofline of the fused kernel (with the DRAM traffic of the committed
ncu capture), the end-to-end rate through the Python API with host copies,
the component kernels, the comparison modes (threshold selection, identity
and folded rotation, sparse + low rank; the threshold and low-rank modes also
at 16 tokens per call), the sparsity and batch sweeps, the other workloads
(a 32-layer 7B stack and an 8-layer 70B slice, each with the dense GEMV and
the folded path; a 13B layer at 1 to 16 tokens), a pure-read probe, clocks and
the CPU oracle's rate.  ``--impl reference`` times the fp64 CPU oracle on the
same workload instead (the only other path that may run it here).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "rotated-sparse linear tokens/s & HBM GB/s (% of roofline), LLaMA2-7B shapes, 40% sparse"
UNIT = "tokens/s"
HIDDEN, FFN, KV = 4096, 11008, 4096
WORKLOAD_ID = 1
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=("larosa", "reference"), default="larosa")
    ap.add_argument("--sparsity", type=float, default=40.0)
    ap.add_argument("--cpu-tokens", type=int, default=4,
                    help="tokens in the CPU oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-model-configs", action="store_true",
                    help="skip the 32-layer 7B stack, the 13B batch sweep and the 70B slice")
    a = ap.parse_args(argv)
    if a.warmup < 3:
        ap.error("--warmup must be at least 3")
    return a


# ---------------------------------------------------------------- ranks

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world: int, backend: str):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def reduce_max(value: float, world: int, device=None) -> float:
    """Maximum of a per-rank scalar over all ranks (identity for one rank)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None:
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def aggregate(per_rank_seconds: float, tokens_per_rank: int, world: int, device=None) -> tuple[float, float]:
    """(whole-job tokens/s, slowest rank's seconds): all ranks' tokens over the max time."""
    t = reduce_max(per_rank_seconds, world, device)
    return tokens_per_rank * world / t, t


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and throttle reasons with nvidia-smi while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines: list[str] = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for name, flag in zip(names, parts[4:8]):
                if flag.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- byte model

def path_bytes(g, K: int, rotate: bool = True) -> dict:
    """Algorithmic HBM bytes of one token through one projection group.

    kept rows K*d_out*2 (bf16), the rotation d_in^2*2 when rotated online,
    and the activations: x (d_in*2), x_rot (d_in*4), idx/val (K*8), y (d_out*4).
    """
    rows = K * g.d_out * 2
    q = g.d_in * g.d_in * 2 if rotate else 0
    act = g.d_in * 2 + g.d_in * 4 + K * 8 + g.d_out * 4
    return {"rows": rows, "q": q, "act": act, "total": rows + q + act}


def measured_peaks() -> tuple[float, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def _code_only(text: str) -> str:
    """C++/CUDA source without its comments, blank lines and trailing spaces."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*$", "", line).rstrip() for line in text.splitlines())
    return "\n".join(line for line in lines if line)


def kernel_source_hash() -> str:
    """Hash of the fused kernel's code (onetoken.cu, common.cuh, select.cuh),
    comments excluded: a stored ncu capture stays valid while only comments
    change, and is dropped as soon as the code does."""
    h = hashlib.sha256()
    for name in ("onetoken.cu", "common.cuh", "select.cuh"):
        with open(os.path.join(ROOT, "activation_sparsity_b200", "csrc", name), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str):
    """DRAM bytes per launch of ``kernel`` from the committed ncu summary, if the
    summary was taken on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    ent = rec.get(kernel)
    if not ent or ent.get("source_hash") != kernel_source_hash():
        return None
    return ent.get("dram_bytes_per_launch")


# ---------------------------------------------------------------- CPU oracle

def cpu_layer_inputs(sparsity: float, seed_layer: int = 0):
    """fp64 host arrays of the 7B layer for the oracle.

    The rotation is a dense orthogonal matrix of the group's size: the
    Kronecker product of two seeded Haar rotations of sizes a x b = d (the
    oracle's cost of applying it is that of any dense d x d matrix, and it is
    built in milliseconds instead of a d x d QR).  The counter-rotated weight
    is drawn directly as N(0, 0.02^2): Q^T W of a Gaussian W is again
    Gaussian with the same law, and the fp64 counter-rotation itself is an
    offline step outside the per-token metric.
    """
    import numpy as np
    import synthdata as sd
    groups = []
    for p in sd.llama_layer(HIDDEN, FFN, KV):
        base = sd.seed_for(WORKLOAD_ID, seed_layer, 10 * p.q_id)
        rng = np.random.default_rng(base + 1)
        a = max(f for f in range(1, int(p.d_in ** 0.5) + 1) if p.d_in % f == 0)
        qa = np.linalg.qr(rng.standard_normal((a, a)))[0]
        qb = np.linalg.qr(rng.standard_normal((p.d_in // a, p.d_in // a)))[0]
        Q = np.kron(qa, qb)
        W_rot = rng.standard_normal((p.d_in, p.d_out)).astype(np.float32).astype(np.float64) * 0.02
        x = sd.activations(1, p.d_in, base + 3, dtype=__import__("torch").float32).double().numpy()
        groups.append((p.name, x, Q, W_rot, sd.k_for_sparsity(p.d_in, sparsity)))
    return groups


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_oracle_seconds_per_token(groups, tokens: int) -> float:
    import oracle
    t0 = time.perf_counter()
    for _ in range(tokens):
        for _, x, Q, W_rot, K in groups:
            oracle.rotate_topk_linear(x, Q, W_rot, K)
    return (time.perf_counter() - t0) / tokens


# ---------------------------------------------------------------- reference arm

def bench_reference(args):
    """The fp64 oracle on the host cores, timed over exactly --steps steps.

    A step is one decode token through the layer's four groups when that
    fits the time budget; for larger --steps each step is a bounded sample
    of a token, so that the whole run stays within a few minutes: per
    group, a block of the rotation's output columns (the oracle's dense
    product x . Q[:, block], the same sums as its rotation) and a block of
    W_rot's output columns (its sparse product on the kept rows), and the
    whole Top-K of the token's rotated vector on as many steps as tokens are
    done.  Tokens are counted as the share of the token's multiply-adds that
    the blocks perform.
    """
    import numpy as np
    import oracle
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    groups = cpu_layer_inputs(args.sparsity)
    t_tok = cpu_oracle_seconds_per_token(groups, 1)  # prices a whole token
    budget_s = 60.0
    frac = min(1.0, budget_s / (max(1, args.steps + args.warmup) * t_tok))
    if frac >= 1.0:
        def step(_i):
            cpu_oracle_seconds_per_token(groups, 1)
        tokens_per_step = 1.0
        sample = ("each step: one decode token through the 4 projection groups of the LLaMA2-7B layer "
                  "(fp64 numpy oracle, rank 0 only)")
    else:
        x_rots = [oracle.rotate(x, Q) for _, x, Q, _, _ in groups]
        blocks = []
        done = total = 0
        for _, x, Q, W_rot, K in groups:
            d, d_out = Q.shape[0], W_rot.shape[1]
            m = min(d, max(8, int(np.ceil(frac * d))))
            n = min(d_out, max(8, int(np.ceil(frac * d_out))))
            blocks.append((m, n))
            done += m * d + K * n
            total += d * d + K * d_out
        tokens_per_step = done / total

        kept = [oracle.topk(xr, K) for xr, (_, _, _, _, K) in zip(x_rots, groups)]

        def step(i):
            # the Top-K (whole) runs on the steps where the count of tokens
            # done passes an integer: as many Top-Ks as tokens
            due = int((i + 1) * tokens_per_step) > int(i * tokens_per_step)
            for g, ((_, x, Q, W_rot, K), xr, (m, n)) in enumerate(zip(groups, x_rots, blocks)):
                c0 = (i * m) % (Q.shape[1] - m + 1)
                o0 = (i * n) % (W_rot.shape[1] - n + 1)
                oracle.dense_linear(x, Q[:, c0:c0 + m])
                if due:
                    kept[g] = oracle.topk(xr, K)
                idx, val = kept[g]
                oracle.sparse_linear(idx, val, W_rot[:, o0:o0 + n])
        sample = (f"each step: {tokens_per_step:.4g} of a decode token through the 4 projection groups of "
                  "the LLaMA2-7B layer: per group a block of the rotation's output columns and of "
                  "W_rot's output columns, and the whole Top-K on as many steps as tokens are done; "
                  "tokens counted as the share of the token's multiply-adds done "
                  "(fp64 numpy oracle, rank 0 only)")
    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    dt = time.perf_counter() - t0
    value = args.steps * tokens_per_step / dt
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": workload_config(args.sparsity, graph=False),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(sparsity: float, graph: bool) -> dict:
    return {
        "workload": "llama2-7b-layer: one decoder layer, batch 1 decode, q|k|v 4096x12288, o 4096x4096, "
                    "gate|up 4096x22016, down 11008x4096, one orthogonal rotation per input "
                    "(3 x 4096^2 + 11008^2), bf16 weights, fp32 accumulate",
        "sparsity_pct": sparsity,
        "batch_tokens": 1,
        "l2": "inputs larger than L2: 586 MB of rotations and kept rows per step vs 126 MB L2, no flush",
        "cuda_graph": graph,
    }


# ---------------------------------------------------------------- the other workloads

class PerfGroup:
    """One projection group of a perf-only layer (no dense weight kept)."""

    def __init__(self, name, d_in, d_out, Qt, W_rot, x):
        self.name, self.d_in, self.d_out = name, d_in, d_out
        self.Qt, self.W_rot, self.x = Qt, W_rot, x


def perf_layers(torch, sd, hidden: int, ffn: int, kv: int, n_layers: int, workload_id: int, M: int,
                device) -> list:
    """``n_layers`` decoder layers of distinct, device-resident tensors.

    Rotations: one seeded Haar rotation per input width (fp32 QR on the
    device, rounded to bf16), and for every layer and group a seeded signed
    permutation of its rows, which is again orthogonal.  W_rot is drawn
    directly as N(0, 0.02^2): for a Gaussian W, Q^T W has that distribution.
    Activations are the heavy-tailed rows of the single-layer workload.
    """
    projs = sd.llama_layer(hidden, ffn, kv)
    gen = torch.Generator(device=device)
    gen.manual_seed(sd.seed_for(workload_id, 999, 0))
    base = {}
    for p in projs:
        if p.d_in not in base:
            base[p.d_in] = sd.orthogonal(p.d_in, sd.seed_for(workload_id, 999, p.d_in % 997),
                                         device=device).to(torch.bfloat16)
    layers = []
    for layer in range(n_layers):
        gs = []
        for p in projs:
            perm = torch.randperm(p.d_in, generator=gen, device=device)
            sign = torch.randint(0, 2, (p.d_in, 1), generator=gen, device=device).to(torch.bfloat16) * 2 - 1
            Qt = (base[p.d_in][perm] * sign).contiguous()
            W_rot = torch.randn((p.d_in, p.d_out), generator=gen, device=device, dtype=torch.float32)
            W_rot = W_rot.mul_(0.02).to(torch.bfloat16)
            x = sd.activations(M, p.d_in, sd.seed_for(workload_id, layer, 10 * p.q_id + 3), torch.bfloat16,
                               device=device)
            gs.append(PerfGroup(p.name, p.d_in, p.d_out, Qt, W_rot, x))
        layers.append(gs)
    del base
    if torch.device(device).type == "cuda":
        torch.cuda.synchronize(device)
    return layers


def bench_model_configs(args, torch, L, sd, device, stream, world, graph_of, time_graph, peak) -> dict:
    """The other workloads of the path, each with its own device-resident tensors.

    * llama2-7b-stack: 32 decoder layers (128 fused calls per token), at 0,
      25, 40 and 50 % sparsity, from a CUDA graph and from eager launches;
      the library's dense bf16 GEMV over the same stack; microseconds per
      projection group (one group's 32 calls back to back);
    * llama2-13b-layer: the fused path with M = 1, 2, 4, 8, 16 tokens per
      call, each token its own Top-K (bytes: Q once plus the union of kept rows);
    * llama2-70b-slice: 8 layers (q|k|v 8192x10240 with GQA, ffn 28672) at 40
      and 50 %, with the rotation online and folded into the producer (the
      identity rotation on an input that arrives rotated), and the dense GEMV.
    The 7B stack also runs the folded path at 40 %.
    Each is timed over a short run (inputs far larger than L2) and freed
    before the next is built.
    """
    st = torch.zeros(1, dtype=torch.int32, device=device)
    n = max(10, min(100, args.steps // 30))
    out = {}
    t0 = time.time()

    def log(msg):
        print(f"[bench] {msg}: {time.time() - t0:.1f} s", file=sys.stderr, flush=True)

    def time_eager(fn, steps):
        with torch.cuda.stream(stream):
            for _ in range(args.warmup):
                fn()
        torch.cuda.synchronize(device)
        barrier(world, device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(steps):
                fn()
            e1.record(stream)
        torch.cuda.synchronize(device)
        barrier(world, device)
        return e0.elapsed_time(e1) / 1e3

    def rate(t, steps, tokens_per_step, step_bytes):
        tps, t_max = aggregate(t, steps * tokens_per_step, world, device)
        return {"tokens_per_s": tps, "ms_per_token": t_max * 1e3 / (steps * tokens_per_step),
                "gb_per_token": step_bytes / tokens_per_step / 1e9,
                "hbm_frac": step_bytes * steps / t_max / 1e9 / peak}

    def fused_bytes(layers, sp, rotate=True):
        return sum(path_bytes(g, sd.k_for_sparsity(g.d_in, sp), rotate)["total"] for gs in layers for g in gs)

    def dense_bytes(layers):
        return sum(g.d_in * g.d_out * 2 + g.d_in * 2 + g.d_out * 4 for gs in layers for g in gs)

    def presize(ws, layers, Ms=(1,)):
        for g in layers[0]:
            for M in Ms:
                ws.get(M, g.d_in, g.d_out, g.d_in)

    # ---- 7B: 32-layer stack
    layers = perf_layers(torch, sd, 4096, 11008, 4096, 32, 2, 1, device)
    log("7B stack built")
    ws = L.Workspace(device)
    presize(ws, layers)
    ys = {g.name: torch.empty((1, g.d_out), dtype=torch.float32, device=device) for g in layers[0]}

    def stack_step(sp, only=None, folded=False):
        # folded: the rotation folded into the producer, so the input arrives
        # rotated and the call runs with the identity rotation (no Q read)
        Ks = {g.name: sd.k_for_sparsity(g.d_in, sp) for g in layers[0]}

        def step():
            for gs in layers:
                for g in gs:
                    if only is None or g.name == only:
                        L.larosa_rotate_topk_linear(g.x, None if folded else g.Qt, g.W_rot, Ks[g.name],
                                                    y=ys[g.name], ws=ws, dev_status=st)
        return step

    def dense_stack():
        # the dense GEMV reads an nn.Linear-layout [d_out x d_in] weight: each
        # layer's random W_rot buffer serves as one (same bytes, random values)
        for gs in layers:
            for g in gs:
                L.larosa_dense_linear(g.x, g.W_rot.view(g.d_out, g.d_in), y=ys[g.name])

    stack = {"layers": 32, "calls_per_token": 128, "fused": {}}
    for sp in (0.0, 25.0, 40.0, 50.0):
        gr = graph_of(stack_step(sp))
        stack["fused"][f"{sp:g}%"] = rate(time_graph(gr, n, args.warmup)[0], n, 1, fused_bytes(layers, sp))
        del gr
    stack["fused_eager_40%"] = rate(time_eager(stack_step(40.0), n), n, 1, fused_bytes(layers, 40.0))
    gr = graph_of(stack_step(40.0, folded=True))
    stack["folded_40%"] = rate(time_graph(gr, n, args.warmup)[0], n, 1, fused_bytes(layers, 40.0, rotate=False))
    del gr
    gr = graph_of(dense_stack)
    stack["dense"] = rate(time_graph(gr, n, args.warmup)[0], n, 1, dense_bytes(layers))
    del gr
    stack["folded_vs_dense_40%"] = stack["folded_40%"]["tokens_per_s"] / stack["dense"]["tokens_per_s"]
    stack["dense_eager"] = rate(time_eager(dense_stack, n), n, 1, dense_bytes(layers))
    stack["fused_vs_dense_40%"] = stack["fused"]["40%"]["tokens_per_s"] / stack["dense"]["tokens_per_s"]
    us = {}
    for g in layers[0]:
        gr = graph_of(stack_step(40.0, only=g.name))
        t, _ = time_graph(gr, n, args.warmup)
        us[g.name] = reduce_max(t, world, device) / (n * 32) * 1e6
        del gr
    stack["us_per_projection_40%"] = us
    out["llama2-7b-stack"] = stack
    log("7B stack timed")
    del layers, ws, ys
    torch.cuda.empty_cache()

    # ---- 13B: one layer, M tokens per call
    Ms = (1, 2, 4, 8, 16)
    per_M = {M: perf_layers(torch, sd, 5120, 13824, 5120, 1, 3, M, device)[0] for M in Ms}
    ws = L.Workspace(device)
    presize(ws, [per_M[1]], Ms)
    ysM = {M: {g.name: torch.empty((M, g.d_out), dtype=torch.float32, device=device) for g in per_M[M]}
           for M in Ms}
    sweep = {}
    for M in Ms:
        gs = per_M[M]
        Ks = {g.name: sd.k_for_sparsity(g.d_in, 40.0) for g in gs}

        def step(gs=gs, Ks=Ks, M=M):
            for g in gs:
                L.larosa_rotate_topk_linear(g.x, g.Qt, g.W_rot, Ks[g.name], y=ysM[M][g.name], ws=ws,
                                            dev_status=st)
        nbytes = 0
        for g in gs:
            idx, _ = L.larosa_topk(L.larosa_rotate(g.x, g.Qt), Ks[g.name], dev_status=st)
            rows = int(torch.unique(idx.flatten()).numel())
            nbytes += rows * g.d_out * 2 + g.d_in * g.d_in * 2 + M * (g.d_in * 6 + Ks[g.name] * 8 + g.d_out * 4)
        gr = graph_of(step)
        sweep[f"M={M}"] = rate(time_graph(gr, n, args.warmup)[0], n, M, nbytes)
        del gr
    out["llama2-13b-layer"] = {"batch_sweep_40%": sweep}
    log("13B layer timed")
    del per_M, ws, ysM
    torch.cuda.empty_cache()

    # ---- 70B: 8-layer slice
    layers = perf_layers(torch, sd, 8192, 28672, 1024, 8, 4, 1, device)
    log("70B slice built")
    ws = L.Workspace(device)
    presize(ws, layers)
    ys = {g.name: torch.empty((1, g.d_out), dtype=torch.float32, device=device) for g in layers[0]}
    slc = {"layers": 8, "fused": {}, "folded": {}}
    for sp in (40.0, 50.0):
        gr = graph_of(stack_step(sp))
        slc["fused"][f"{sp:g}%"] = rate(time_graph(gr, n, args.warmup)[0], n, 1, fused_bytes(layers, sp))
        del gr
        gr = graph_of(stack_step(sp, folded=True))
        slc["folded"][f"{sp:g}%"] = rate(time_graph(gr, n, args.warmup)[0], n, 1,
                                          fused_bytes(layers, sp, rotate=False))
        del gr
    gr = graph_of(dense_stack)
    slc["dense"] = rate(time_graph(gr, n, args.warmup)[0], n, 1, dense_bytes(layers))
    del gr
    for sp in ("40%", "50%"):
        slc[f"folded_vs_dense_{sp}"] = slc["folded"][sp]["tokens_per_s"] / slc["dense"]["tokens_per_s"]
    out["llama2-70b-slice"] = slc
    log("70B slice timed")
    del layers, ws, ys
    torch.cuda.empty_cache()
    assert L.larosa_check(st, device=device) == 0
    out["timed_steps"] = n
    return out


def read_probe(torch, L, device, stream, warmup: int) -> dict:
    """Pure-read bandwidth: the library's dense GEMV over a 4 GiB bf16 weight
    (one token: the weight is the whole traffic) and torch's sum of the same
    buffer, each timed with CUDA events over 10 passes."""
    d_in, d_out = 32768, 65536
    W = torch.empty((d_out, d_in), dtype=torch.bfloat16, device=device).normal_()
    x = torch.ones((1, d_in), dtype=torch.bfloat16, device=device)
    y = torch.empty((1, d_out), dtype=torch.float32, device=device)
    res = {}
    for name, fn in (("dense_gemv_gbs", lambda: L.larosa_dense_linear(x, W, y=y)),
                     ("torch_sum_gbs", lambda: torch.sum(W, dtype=torch.float32))):
        with torch.cuda.stream(stream):
            for _ in range(warmup):
                fn()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(10):
                fn()
            e1.record(stream)
        torch.cuda.synchronize(device)
        res[name] = W.numel() * 2 * 10 / (e0.elapsed_time(e1) / 1e3) / 1e9
    del W
    torch.cuda.empty_cache()
    res["bytes"] = d_in * d_out * 2
    return res


# ---------------------------------------------------------------- larosa arm

def bench_larosa(args):
    import numpy as np
    import torch

    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device (the library has no CPU path)")
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    init_dist(world, "nccl")

    import activation_sparsity_b200 as L
    import synthdata as sd
    from activation_sparsity_b200.workload import build_layer

    layer = build_layer(HIDDEN, FFN, KV, args.sparsity, WORKLOAD_ID, layer=rank, device=device)
    groups = layer.groups
    stream = torch.cuda.Stream(device)
    ws = L.Workspace(device)
    # size the workspace once for every call below (one token up to 16, Top-K
    # and threshold), so that no captured graph holds a buffer that a later
    # call would replace
    for g in groups:
        for M in (1, 2, 4, 8, 16):
            ws.get(M, g.d_in, g.d_out, g.d_in)
            ws.get(M, g.d_in, g.d_out, g.K)
    st = torch.zeros(1, dtype=torch.int32, device=device)
    ys = [torch.empty((1, g.d_out), dtype=torch.float32, device=device) for g in groups]
    for g in groups:
        ws.get(1, g.d_in, g.d_out, g.d_in)
    # component-call intermediates for the per-kernel pass
    x_rots = [torch.empty((1, g.d_in), dtype=torch.float32, device=device) for g in groups]
    idxs = [torch.empty((1, g.K), dtype=torch.int32, device=device) for g in groups]
    vals = [torch.empty((1, g.K), dtype=torch.float32, device=device) for g in groups]

    def fused_step():
        for g, y in zip(groups, ys):
            L.larosa_rotate_topk_linear(g.x, g.Qt, g.W_rot, g.K, y=y, ws=ws, dev_status=st)

    def rotate_step():
        for g, xr in zip(groups, x_rots):
            L.larosa_rotate(g.x, g.Qt, x_rot=xr)

    # the other sparsities of the sweep (same layer, K from the sparsity) and
    # batches of M tokens (each keeps its own Top-K; the rows kept by any
    # token are streamed once)
    sweep = (0.0, 25.0, 50.0)
    batch_sizes = (2, 4, 8, 16)
    x_batch = {M: [sd.activations(M, g.d_in, sd.seed_for(WORKLOAD_ID, 900 + M, 10 * gi + 3),
                                  torch.bfloat16, device=device) for gi, g in enumerate(groups)]
               for M in batch_sizes}
    y_batch = {M: [torch.empty((M, g.d_out), dtype=torch.float32, device=device) for g in groups]
               for M in batch_sizes}

    def sparsity_step(sp):
        Ks = [sd.k_for_sparsity(g.d_in, sp) for g in groups]

        def step():
            for g, y, K in zip(groups, ys, Ks):
                L.larosa_rotate_topk_linear(g.x, g.Qt, g.W_rot, K, y=y, ws=ws, dev_status=st)
        return step

    def batch_step(M):
        def step():
            for g, x, y in zip(groups, x_batch[M], y_batch[M]):
                L.larosa_rotate_topk_linear(x, g.Qt, g.W_rot, g.K, y=y, ws=ws, dev_status=st)
        return step

    def rotate_topk_step():  # the fused path's first kernel: rotation, then Top-K by its last CTA
        for gi, g in enumerate(groups):
            L.larosa_rotate_topk(g.x, g.Qt, g.K, x_rot=x_rots[gi], idx=idxs[gi], val=vals[gi], ws=ws,
                                 dev_status=st)

    def topk_step():
        for gi, g in enumerate(groups):
            L.larosa_topk(x_rots[gi], g.K, idx=idxs[gi], val=vals[gi], dev_status=st)

    def gather_step():
        for gi, g in enumerate(groups):
            L.larosa_sparse_linear(idxs[gi], vals[gi], g.W_rot, y=ys[gi], ws=ws, dev_status=st)

    def sparse_only_step():  # the same path on pre-rotated inputs (no Q streamed): Top-K + sparse linear
        for gi, g in enumerate(groups):
            L.larosa_topk_linear(x_rots[gi], g.W_rot, g.K, y=ys[gi], ws=ws, dev_status=st)

    def dense_step():
        for g, y in zip(groups, ys):
            L.larosa_dense_linear(g.x, g.Wt, y=y)

    # comparison modes: the unrotated fixed-K path (Q = I, plain weight) and the
    # threshold selection |x_rot| >= t, rotated and unrotated, with t set per
    # group from this token's own magnitudes so that the same share is dropped
    def unrot_topk_step():
        for g, y in zip(groups, ys):
            L.larosa_rotate_topk_linear(g.x, None, g.W, g.K, y=y, ws=ws, dev_status=st)

    def rot_thr_step():
        for gi, (g, y) in enumerate(zip(groups, ys)):
            L.larosa_rotate_threshold_linear(g.x, g.Qt, g.W_rot, t_rot[gi], y=y, ws=ws, dev_status=st)

    def batch_thr_step():  # 16 tokens per call with the threshold selection
        for gi, (g, x, y) in enumerate(zip(groups, x_batch[16], y_batch[16])):
            L.larosa_rotate_threshold_linear(x, g.Qt, g.W_rot, t_rot[gi], y=y, ws=ws, dev_status=st)

    def unrot_thr_step():
        for gi, (g, y) in enumerate(zip(groups, ys)):
            L.larosa_rotate_threshold_linear(g.x, None, g.W, t_x[gi], y=y, ws=ws, dev_status=st)

    # the rotation folded into the producer: the input arrives rotated (as the
    # producer's bf16 output x . Q) and the call runs with the identity rotation
    def folded_topk_step():
        for gi, (g, y) in enumerate(zip(groups, ys)):
            L.larosa_rotate_topk_linear(x_folded[gi], None, g.W_rot, g.K, y=y, ws=ws, dev_status=st)

    # sparse + low-rank compensation of the dropped entries (rank-256
    # factors of each group's weight, random here: the time depends on shapes)
    LR = 256
    lr_A = [sd.weights(g.d_in, LR, 0.02, sd.seed_for(WORKLOAD_ID, 950, 10 * gi + 1), torch.bfloat16, device=device)
            for gi, g in enumerate(groups)]
    lr_B = [sd.weights(LR, g.d_out, 0.02, sd.seed_for(WORKLOAD_ID, 950, 10 * gi + 2), torch.bfloat16, device=device)
            for gi, g in enumerate(groups)]
    lr_ws = [torch.zeros(L.larosa_lowrank_workspace_bytes(1, g.d_in, g.d_out, g.K, LR), dtype=torch.uint8,
                         device=device) for g in groups]

    def lowrank_step():
        for gi, (g, y) in enumerate(zip(groups, ys)):
            L.larosa_sparse_lowrank_linear(x_rots[gi], idxs[gi], vals[gi], g.W_rot, lr_A[gi], lr_B[gi], y=y,
                                           ws=lr_ws[gi], dev_status=st)

    # the same mode with 16 tokens per call (pre-rotated inputs, their Top-K lists)
    lr_x16 = [L.larosa_rotate(x, g.Qt) for g, x in zip(groups, x_batch[16])]
    lr_sel16 = [L.larosa_topk(xr, g.K, dev_status=st) for g, xr in zip(groups, lr_x16)]
    lr_ws16 = [torch.zeros(L.larosa_lowrank_workspace_bytes(16, g.d_in, g.d_out, g.K, LR), dtype=torch.uint8,
                           device=device) for g in groups]

    def lowrank16_step():
        for gi, (g, y) in enumerate(zip(groups, y_batch[16])):
            L.larosa_sparse_lowrank_linear(lr_x16[gi], lr_sel16[gi][0], lr_sel16[gi][1], g.W_rot, lr_A[gi],
                                           lr_B[gi], y=y, ws=lr_ws16[gi], dev_status=st)

    def folded_thr_step():
        for gi, (g, y) in enumerate(zip(groups, ys)):
            L.larosa_rotate_threshold_linear(x_folded[gi], None, g.W_rot, t_rot[gi], y=y, ws=ws,
                                             dev_status=st)

    def graph_of(fn):
        with torch.cuda.stream(stream):
            for _ in range(3):
                fn()
        torch.cuda.synchronize(device)
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream):
            fn()
        torch.cuda.synchronize(device)
        return gr

    def time_graph(gr, steps: int, warmup: int, clocks: ClockSampler | None = None):
        with torch.cuda.stream(stream):
            for _ in range(warmup):
                gr.replay()
        torch.cuda.synchronize(device)
        barrier(world, device)
        if clocks:
            clocks.start()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(steps):
                gr.replay()
            e1.record(stream)
        torch.cuda.synchronize(device)
        clk = clocks.stop() if clocks else None
        barrier(world, device)
        return e0.elapsed_time(e1) / 1e3, clk

    # rotate and select once so the component graphs have their inputs
    with torch.cuda.stream(stream):
        rotate_step()
        topk_step()
    torch.cuda.synchronize(device)

    def calibrate(mag: torch.Tensor, d: int) -> tuple[float, int]:
        """t = the magnitude below which the sparsity's share of entries lies; kept count."""
        srt = torch.sort(mag.flatten().float()).values
        t = float(srt[d - sd.k_for_sparsity(d, args.sparsity)].item())
        return t, int((mag >= t).sum().item())
    x_folded = [xr.to(torch.bfloat16) for xr in x_rots]
    t_rot, nnz_rot, t_x, nnz_x = [], [], [], []
    for gi, g in enumerate(groups):
        t, n = calibrate(x_rots[gi].abs(), g.d_in)
        t_rot.append(t)
        nnz_rot.append(n)
        t, n = calibrate(g.x.float().abs(), g.d_in)
        t_x.append(t)
        nnz_x.append(n)
    t_rot_list = list(t_rot)  # (t_rot is reused for a time below)

    g_fused = graph_of(fused_step)
    g_sparse = graph_of(sparse_only_step)
    g_dense = graph_of(dense_step)
    g_rot = graph_of(rotate_step)
    g_rotsel = graph_of(rotate_topk_step)
    g_topk = graph_of(topk_step)
    g_gather = graph_of(gather_step)
    g_unrot_topk = graph_of(unrot_topk_step)
    g_rot_thr = graph_of(rot_thr_step)
    g_unrot_thr = graph_of(unrot_thr_step)
    g_folded_topk = graph_of(folded_topk_step)
    g_sweep = {sp: graph_of(sparsity_step(sp)) for sp in sweep}
    g_batch = {M: graph_of(batch_step(M)) for M in batch_sizes}
    g_batch_thr = graph_of(batch_thr_step)
    g_folded_thr = graph_of(folded_thr_step)
    g_lowrank = graph_of(lowrank_step)
    g_lowrank16 = graph_of(lowrank16_step)

    props = torch.cuda.get_device_properties(device)
    clocks = ClockSampler(f"GPU-{props.uuid}")
    t_fused, clk = time_graph(g_fused, args.steps, args.warmup, clocks)
    value, t_max = aggregate(t_fused, args.steps, world, device)
    t_sparse, _ = time_graph(g_sparse, args.steps, args.warmup)
    t_dense, _ = time_graph(g_dense, args.steps, args.warmup)
    sparse_tps, _ = aggregate(t_sparse, args.steps, world, device)
    dense_tps, _ = aggregate(t_dense, args.steps, world, device)

    # ---- per-kernel pass: graphs holding one kernel type for the four groups,
    # timed with CUDA events on the launching stream over the same steps
    t_rot, _ = time_graph(g_rot, args.steps, args.warmup)
    t_rotsel, _ = time_graph(g_rotsel, args.steps, args.warmup)
    t_topk, _ = time_graph(g_topk, args.steps, args.warmup)
    t_gather, _ = time_graph(g_gather, args.steps, args.warmup)
    t_unrot_topk, _ = time_graph(g_unrot_topk, args.steps, args.warmup)
    t_rot_thr, _ = time_graph(g_rot_thr, args.steps, args.warmup)
    t_unrot_thr, _ = time_graph(g_unrot_thr, args.steps, args.warmup)
    t_folded_topk, _ = time_graph(g_folded_topk, args.steps, args.warmup)
    t_folded_thr, _ = time_graph(g_folded_thr, args.steps, args.warmup)
    t_lowrank, _ = time_graph(g_lowrank, args.steps, args.warmup)
    t_lowrank16 = time_graph(g_lowrank16, max(1, args.steps // 4), args.warmup)[0]
    side_steps = max(1, args.steps // 4)
    t_sweep = {sp: time_graph(gr, side_steps, args.warmup)[0] for sp, gr in g_sweep.items()}
    t_batch = {M: time_graph(gr, side_steps, args.warmup)[0] for M, gr in g_batch.items()}
    t_batch_thr = time_graph(g_batch_thr, side_steps, args.warmup)[0]
    # rows streamed per batch step: the union of the tokens' kept rows (Q once per batch)
    batch_bytes = {}
    for M in batch_sizes:
        tot = 0
        for g, x in zip(groups, x_batch[M]):
            xr = L.larosa_rotate(x, g.Qt)
            idx, _ = L.larosa_topk(xr, g.K, dev_status=st)
            rows = int(torch.unique(idx.flatten()).numel())
            tot += rows * g.d_out * 2 + g.d_in * g.d_in * 2 + M * (g.d_in * 6 + g.K * 8 + g.d_out * 4)
        batch_bytes[M] = tot
    # the 16-token threshold step: Q once, the union of the kept rows
    batch_thr_bytes = 0
    for gi, (g, x) in enumerate(zip(groups, x_batch[16])):
        xr = L.larosa_rotate(x, g.Qt)
        idx, _, nnz = L.larosa_threshold(xr, t_rot_list[gi], dev_status=st)
        kept = torch.cat([idx[m, :int(nnz[m].item())] for m in range(16)])
        rows = int(torch.unique(kept).numel())
        batch_thr_bytes += (rows * g.d_out * 2 + g.d_in * g.d_in * 2 + 16 * (g.d_in * 6 + g.d_out * 4)
                            + int(nnz.sum().item()) * 8)
    n_launch = args.steps * len(groups)
    rot_us = t_rot / n_launch * 1e6
    rotsel_us = t_rotsel / n_launch * 1e6
    topk_us = t_topk / n_launch * 1e6
    gather_us = t_gather / n_launch * 1e6
    assert L.larosa_check(st, device=device) == 0

    rot_bytes = [g.d_in * g.d_in * 2 + g.d_in * 2 + g.d_in * 4 for g in groups]
    # rotation + Top-K: Q, x, x_rot written and read back once, idx/val written
    rotsel_bytes = [g.d_in * g.d_in * 2 + g.d_in * 2 + 2 * g.d_in * 4 + g.K * 8 for g in groups]
    lin_bytes = [g.K * g.d_out * 2 + g.K * 8 + g.d_out * 4 for g in groups]
    step_bytes = sum(path_bytes(g, g.K)["total"] for g in groups)
    sparse_bytes = sum(path_bytes(g, g.K, rotate=False)["total"] for g in groups)
    lowrank_bytes = sparse_bytes + sum((g.d_in + g.d_out) * LR * 2 + g.d_in * 4 for g in groups)
    lowrank16_bytes = 0
    for g, (idx16, _) in zip(groups, lr_sel16):
        rows = int(torch.unique(idx16.flatten()).numel())
        lowrank16_bytes += (rows * g.d_out * 2 + (g.d_in + g.d_out) * LR * 2
                            + 16 * (g.d_in * 4 + g.K * 8 + g.d_out * 4))
    dense_bytes = sum(g.d_in * g.d_out * 2 + g.d_in * 2 + g.d_out * 4 for g in groups)
    unrot_topk_bytes = sum(path_bytes(g, g.K, rotate=False)["total"] for g in groups)
    rot_thr_bytes = sum(path_bytes(g, n)["total"] for g, n in zip(groups, nnz_rot))
    unrot_thr_bytes = sum(path_bytes(g, n, rotate=False)["total"] for g, n in zip(groups, nnz_x))
    peak, peak_kind = measured_peaks()
    rot_gbs = sum(rot_bytes) * args.steps / t_rot / 1e9
    rotsel_gbs = sum(rotsel_bytes) * args.steps / t_rotsel / 1e9
    lin_gbs = sum(lin_bytes) * args.steps / t_gather / 1e9
    fused_us = t_fused / n_launch * 1e6  # one fused kernel per group
    fused_gbs = step_bytes * args.steps / t_fused / 1e9
    traffic = profiled_traffic("fused")

    # ---- end to end through the public API with host buffers
    # the four groups' inputs live in one pinned host buffer and one device
    # buffer, so a step moves them in with one copy; each group's output is
    # read back on a copy stream as soon as its call is done, while the next
    # group computes, and the step ends when every output is on the host
    x_sizes = [g.x.numel() for g in groups]
    y_sizes = [g.d_out for g in groups]
    x_host_all = torch.cat([g.x.flatten().cpu() for g in groups]).pin_memory()
    x_dev_all = torch.empty_like(x_host_all, device=device)
    x_dev = [v.view(1, -1) for v in torch.split(x_dev_all, x_sizes)]
    y_dev_all = torch.empty(sum(y_sizes), dtype=torch.float32, device=device)
    y_dev = [v.view(1, -1) for v in torch.split(y_dev_all, y_sizes)]
    y_host_all = torch.empty(sum(y_sizes), dtype=torch.float32).pin_memory()
    y_host = list(torch.split(y_host_all, y_sizes))
    copy_stream = torch.cuda.Stream(device)
    done = [torch.cuda.Event() for _ in groups]
    e2e_steps = max(20, min(500, args.steps // 10))
    with torch.cuda.stream(stream):
        for r in range(args.warmup + e2e_steps):
            if r == args.warmup:
                torch.cuda.synchronize(device)
                barrier(world, device)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
            # the step's inputs in, the four groups back to back, each output out
            x_dev_all.copy_(x_host_all, non_blocking=True)
            for gi, g in enumerate(groups):
                L.larosa_rotate_topk_linear(x_dev[gi], g.Qt, g.W_rot, g.K, y=y_dev[gi], ws=ws, dev_status=st)
                done[gi].record(stream)
                copy_stream.wait_event(done[gi])
                with torch.cuda.stream(copy_stream):
                    y_host[gi].copy_(y_dev[gi].view(-1), non_blocking=True)
            stream.wait_stream(copy_stream)  # the step's outputs are on the host
        e1.record(stream)
    torch.cuda.synchronize(device)
    t_e2e = e0.elapsed_time(e1) / 1e3
    e2e_value, _ = aggregate(t_e2e, e2e_steps, world, device)
    assert torch.isfinite(y_host_all).all()

    # ---- the other workloads and the pure-read probe
    model_cfgs = None
    if not args.no_model_configs:
        model_cfgs = bench_model_configs(args, torch, L, sd, device, stream, world, graph_of, time_graph, peak)
    probe = read_probe(torch, L, device, stream, args.warmup)

    # ---- CPU oracle baseline (rank 0, one GPU only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cgroups = cpu_layer_inputs(args.sparsity)
        cpu_oracle_seconds_per_token(cgroups, 1)
        spt = cpu_oracle_seconds_per_token(cgroups, args.cpu_tokens)
        cpu = {"value": 1.0 / spt, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": f"{args.cpu_tokens} decode tokens through the 4 projection groups of the "
                         "LLaMA2-7B layer, fp64 numpy oracle on the host cores"}

    if rank == 0:
        ms_step = t_max * 1e3 / args.steps
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(args.sparsity, graph=True),
            "hbm_gbs": step_bytes / (ms_step * 1e-3) / 1e9,
            "hbm_frac": step_bytes / (ms_step * 1e-3) / 1e9 / peak,
            "bytes_per_step": step_bytes,
            "roofline": {"kernel": "fused_kernel (rotation, Top-K and gather of one projection group "
                                   "in one cooperative launch; bf16)",
                         "bound": "hbm", "achieved": fused_gbs, "peak": peak, "peak_kind": peak_kind,
                         "unit": "GB/s", "frac": fused_gbs / peak, "traffic": traffic,
                         "frac_of_nominal_8tbs": fused_gbs / 8000.0,
                         "algorithmic_bytes_per_launch": step_bytes / len(groups),
                         "avg_launch_us": fused_us, "share_of_step": 1.0},
            "kernels": {
                "fused_us_per_launch": fused_us,
                "rotate_topk_us_per_launch": rotsel_us,
                "rotate_topk_gbs": rotsel_gbs,
                "rotate_only_us_per_launch": rot_us, "rotate_only_gbs": rot_gbs,
                "gather_us_per_launch": gather_us,
                "gather_gbs": lin_gbs, "gather_frac": lin_gbs / peak,
                "topk_us_per_launch": topk_us,
                "groups": [g.name for g in groups],
            },
            "paths": {
                "fused_tokens_per_s": value,
                "sparse_only_tokens_per_s": sparse_tps,
                "sparse_only_hbm_frac": sparse_bytes * sparse_tps / world / 1e9 / peak,
                "dense_tokens_per_s": dense_tps,
                "dense_hbm_frac": dense_bytes * dense_tps / world / 1e9 / peak,
                "sparse_only_vs_dense": sparse_tps / dense_tps,
                # the sparse linear alone on given kept lists (no Q, no Top-K)
                "gather_only_tokens_per_s": args.steps / t_gather * world,
                "gather_only_vs_dense": (args.steps / t_gather * world) / dense_tps,
                "fused_vs_dense": value / dense_tps,
                # comparison modes, each one call per group through the public API
                "unrotated_topk_tokens_per_s": args.steps / t_unrot_topk * world,
                "unrotated_topk_hbm_frac": unrot_topk_bytes * args.steps / t_unrot_topk / 1e9 / peak,
                "rotated_threshold_tokens_per_s": args.steps / t_rot_thr * world,
                "rotated_threshold_hbm_frac": rot_thr_bytes * args.steps / t_rot_thr / 1e9 / peak,
                "rotated_threshold_kept_frac": sum(nnz_rot) / sum(g.d_in for g in groups),
                # 16 tokens per call, each group's t as above (tokens/s counts every token)
                "rotated_threshold_M16_tokens_per_s": 16 * side_steps / t_batch_thr * world,
                "rotated_threshold_M16_hbm_frac": batch_thr_bytes * side_steps / t_batch_thr / 1e9 / peak,
                "unrotated_threshold_tokens_per_s": args.steps / t_unrot_thr * world,
                "unrotated_threshold_hbm_frac": unrot_thr_bytes * args.steps / t_unrot_thr / 1e9 / peak,
                "unrotated_threshold_kept_frac": sum(nnz_x) / sum(g.d_in for g in groups),
                # Q folded into the producer: no Q streamed per token
                "folded_topk_tokens_per_s": args.steps / t_folded_topk * world,
                "folded_topk_hbm_frac": sparse_bytes * args.steps / t_folded_topk / 1e9 / peak,
                "folded_topk_vs_dense": (args.steps / t_folded_topk * world) / dense_tps,
                "folded_threshold_tokens_per_s": args.steps / t_folded_thr * world,
                "folded_threshold_vs_dense": (args.steps / t_folded_thr * world) / dense_tps,
                # kept rows plus rank-256 compensation of the dropped entries, on
                # the pre-rotated input (Q not streamed)
                "sparse_lowrank_r256_tokens_per_s": args.steps / t_lowrank * world,
                "sparse_lowrank_r256_hbm_frac": lowrank_bytes * args.steps / t_lowrank / 1e9 / peak,
                # 16 tokens per call (tokens/s counts every token; bytes: the union
                # of the tokens' kept rows, both factors once, the activations)
                "sparse_lowrank_r256_M16_tokens_per_s": 16 * max(1, args.steps // 4) / t_lowrank16 * world,
                "sparse_lowrank_r256_M16_hbm_frac": lowrank16_bytes * max(1, args.steps // 4) / t_lowrank16
                / 1e9 / peak,
            },
            # the fused path at the sweep's other sparsities, and with M tokens
            # per call (tokens/s counts every token; bytes: Q once plus the
            # union of the tokens' kept rows), each timed over steps/4
            "sparsity_sweep": {
                f"{sp:g}%": {"tokens_per_s": side_steps / t * world,
                             "hbm_frac": sum(path_bytes(g, sd.k_for_sparsity(g.d_in, sp))["total"] for g in groups)
                             * side_steps / t / 1e9 / peak}
                for sp, t in t_sweep.items()},
            "batch_sweep": {
                f"M={M}": {"tokens_per_s": M * side_steps / t * world,
                           "hbm_frac": batch_bytes[M] * side_steps / t / 1e9 / peak}
                for M, t in t_batch.items()},
            "model_configs": model_cfgs,
            "read_probe": probe,
            "e2e": {"value": e2e_value, "unit": UNIT,
                    "h2d_bytes_per_step": sum(g.x.numel() * g.x.element_size() for g in groups),
                    "d2h_bytes_per_step": sum(g.d_out * 4 for g in groups)},
            "gpu_launches": args.steps * len(groups),  # one fused_kernel per group and step
            "clocks": clk,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    del g_fused, g_sparse, g_dense, g_rot, g_rotsel, g_topk, g_gather, g_unrot_topk, g_rot_thr, g_unrot_thr
    del g_folded_topk, g_folded_thr, g_sweep, g_batch, g_lowrank
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return bench_reference(args)
    return bench_larosa(args)


if __name__ == "__main__":
    sys.exit(main())
