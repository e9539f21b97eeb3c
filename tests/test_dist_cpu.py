"""The multi-rank path of bench.py on CPU: two gloo ranks, each with its own step time, agree on
the slowest rank's time and on the whole-job throughput (weak scaling, no data collective)."""
from __future__ import annotations

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        my_seconds = [0.25, 0.40][rank]
        t_max = bench.max_over_ranks(my_seconds, world, "cpu")
        value = bench.aggregate_tflops(1e12, 10, world, t_max)
        out_q.put((rank, t_max, value))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_aggregate():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(world))
    for rank, t_max, value in res:
        assert t_max == pytest.approx(0.40)
        # 2 ranks x 1e12 FLOP x 10 steps / 0.40 s = 50 TFLOP/s
        assert value == pytest.approx(50.0)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(1.5, 1, "cpu") == 1.5
    assert bench.aggregate_tflops(2e12, 3, 1, 1.5) == pytest.approx(4.0)
