"""The N > 1 path of bench.py on CPU with world size 2 over gloo: replicas
only (each rank runs its own token stream, no collective on the data path),
times reduced as the max over ranks, rank 0 alone runs the reference arm."""
import datetime
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r took (r + 1) ms for the steps and (10 - r) ms end to end
        got = bench.max_over_ranks([float(rank + 1), 10.0 - rank])
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world_2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # every rank sees the slowest rank's times
    assert res[0] == res[1] == [2.0, 10.0]


def test_max_over_ranks_without_group_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks([3.5, 1.0]) == [3.5, 1.0]


def test_reference_arm_runs_on_rank_0_only():
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        config = "decode"
        steps = 1
        warmup = 3

    assert bench.run_reference(Args(), rank=1) is None
