"""Host logic of bench.py's multi-rank path with world-size-2 gloo ranks on the
CPU: the device time is the max over ranks and the value is the work of all
ranks over that time.  No GPU involved."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ms = [10.0, 25.0][rank]                    # per-rank device time
        value, ms_max = bench.aggregate(1.5, ms, world)
        q.put((rank, value, ms_max))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_aggregate_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    out = sorted(q.get(timeout=5) for _ in range(2))
    for rank, value, ms_max in out:
        assert ms_max == 25.0                      # the slowest rank's time
        assert value == pytest.approx(1.5 * 2 / 0.025)   # both ranks' units / that time


def test_single_rank_aggregate_is_plain_ratio():
    value, ms = bench.aggregate(3.0, 2.0, 1)
    assert ms == 2.0 and value == pytest.approx(1500.0)
