"""The multi-rank host logic of bench.py on CPU: two gloo ranks (one process
each, rendezvous on 127.0.0.1) check that every reported time is the slowest
rank's and that the whole-job value counts the work of every replica. The
prefill path has no exchange step, so nothing else crosses ranks."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = [3.0, 5.0][rank]            # rank 1 is the slow one
        t = bench.rank_max(local_ms, world, "cpu")
        v = bench.job_value(2.0e12, 10, world, t)
        out.put((rank, t, v))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_job_value():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(out.get(timeout=10) for _ in range(2))
    for rank, t, v in res:
        assert t == 5.0                              # the slowest rank's time
        # 2 replicas x 10 steps x 2e12 ops in 5 ms = 8000 TOPS
        assert v == pytest.approx(2 * 10 * 2.0e12 / 5e-3 / 1e12)


def test_single_rank_is_identity():
    import bench
    assert bench.rank_max(1.25, 1, "cpu") == 1.25
    assert bench.job_value(1e12, 4, 1, 2.0) == pytest.approx(4 * 1e12 / 2e-3 / 1e12)
