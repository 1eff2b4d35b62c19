"""The multi-GPU bench path is replicas with one cross-rank reduction of the
elapsed time. Checked here with two gloo ranks on the CPU (no GPU)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, q):
    import sys
    from datetime import timedelta

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench

    # each rank times its own replica; the job takes as long as the slowest
    ms = [12.5, 20.0][rank]
    ms_max = bench.max_over_ranks(ms)
    value = bench.throughput(128, 10, world, ms_max)
    q.put((rank, ms_max, value))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_max_and_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[1] for o in out] == [20.0, 20.0]
    # 2 ranks x 10 steps x 128 queries in 20 ms
    assert out[0][2] == pytest.approx(2 * 10 * 128 / 0.020)
    assert out[0][2] == out[1][2]


def test_single_process_is_identity():
    import sys

    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.throughput(128, 5, 1, 10.0) == pytest.approx(64000.0)
