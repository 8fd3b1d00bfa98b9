"""The replica timing of bench.py on two CPU ranks (gloo): every rank gets the slowest
rank's time, and the whole-job value counts all ranks' tokens over that time."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        value, ms_max = bench.job_value(8, world, 1.0 + rank, None)
        q.put((rank, value, ms_max))
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, value, ms_max in out:
        assert ms_max == pytest.approx(2.0)            # slowest rank: 1 + 1 ms
        assert value == pytest.approx(8 * 2 / 2.0e-3)  # 16 tokens in 2 ms


def test_single_process_value():
    import bench
    value, ms = bench.job_value(8, 1, 0.5, None)
    assert ms == 0.5 and value == pytest.approx(16000.0)
