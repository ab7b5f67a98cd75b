"""Host logic of the multi-GPU benchmark, run as two gloo ranks on the CPU.

The path does not shard: N GPUs run N independent replicas with no data-path
collective.  What needs checking is the timing aggregation: the whole-job
value is all ranks' tokens over the slowest rank's time.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    bench.init_dist(world, "gloo")
    secs = [0.5, 2.0][rank]
    value, t = bench.aggregate(secs, tokens_per_rank=100, world=world)
    m = bench.reduce_max(float(rank), world)
    bench.barrier(world)
    out.put((rank, value, t, m))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_two_rank_aggregation_uses_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, value, t, m in got:
        assert t == pytest.approx(2.0)
        assert value == pytest.approx(200 / 2.0)
        assert m == 1.0


def test_single_rank_is_identity():
    import bench
    value, t = bench.aggregate(0.25, tokens_per_rank=10, world=1)
    assert t == 0.25 and value == pytest.approx(40.0)
