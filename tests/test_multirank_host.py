"""The multi-rank host logic of bench.py on CPU: two gloo ranks (one process
each, rendezvous on 127.0.0.1) check that every reported time is the slowest
rank's, that the whole-job value counts the whole workload, and that the
kv-head shards of the ranks cover every head exactly once. The prefill path
has no exchange step, so nothing else crosses ranks."""
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
        v = bench.job_value(2.0e12, 10, t)
        # every rank's kv-head shard of a 40-head workload, gathered on all
        lo, hi = bench.kv_head_range(40, world, rank)
        ranges = [None] * world
        dist.all_gather_object(ranges, (lo, hi))
        out.put((rank, t, v, ranges))
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
    for rank, t, v, ranges in res:
        assert t == 5.0                              # the slowest rank's time
        # 10 steps x 2e12 ops of the whole workload in 5 ms = 4000 TOPS
        assert v == pytest.approx(10 * 2.0e12 / 5e-3 / 1e12)
        heads = [h for lo, hi in ranges for h in range(lo, hi)]
        assert heads == list(range(40))              # every head once, in order


def test_single_rank_is_identity():
    import bench
    assert bench.rank_max(1.25, 1, "cpu") == 1.25
    assert bench.job_value(1e12, 4, 2.0) == pytest.approx(4 * 1e12 / 2e-3 / 1e12)


@pytest.mark.parametrize("Hk,world", [(40, 1), (40, 3), (40, 8), (24, 5), (32, 32), (1, 1)])
def test_kv_head_shards_partition_the_heads(Hk, world):
    import bench
    ranges = [bench.kv_head_range(Hk, world, r) for r in range(world)]
    assert [h for lo, hi in ranges for h in range(lo, hi)] == list(range(Hk))
    sizes = [hi - lo for lo, hi in ranges]
    assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1


def test_shard_heads_keeps_query_groups_with_their_kv_head():
    import torch

    import bench
    cfg = dict(B=1, H=8, Hk=4, L=16, D=64)
    q = torch.arange(8).view(1, 8, 1, 1).expand(1, 8, 16, 64)
    k = torch.arange(4).view(1, 4, 1, 1).expand(1, 4, 16, 64)
    seen = []
    for r in range(2):
        c, qs, ks, vs = bench.shard_heads(cfg, q, k, k, 2, r)
        assert c["H"] == 4 and c["Hk"] == 2
        for j in range(c["H"]):
            # query head h reads kv head h // (H / Hk) of the full tensor
            assert int(qs[0, j, 0, 0]) // 2 == int(ks[0, j // 2, 0, 0])
        seen += qs[0, :, 0, 0].tolist()
    assert seen == list(range(8))
