"""The multi-rank path of bench.py on CPU: two gloo ranks (spawned processes) run the
replica aggregation -- barrier, max of the per-rank device time, sum of the per-rank
bytes -- and the whole-job rate is the bytes of both ranks over the slower rank's time.
The decode path itself has no cross-rank step (replicas only)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist

    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dev = torch.device("cpu")
        ms = [2.0, 3.0][rank]             # rank 1 is the slower replica
        nbytes = [4.0e9, 6.0e9][rank]
        bench.rank_barrier(world)
        gbps, ms_max, total = bench.replica_gbps(nbytes, ms, world, dev)
        out[rank] = (gbps, ms_max, total, bench.rank_reduce(float(rank + 1), world, dev, "sum"))
        bench.rank_barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_gloo_replicas_aggregate():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(out)
    for r in range(2):
        gbps, ms_max, total, s = res[r]
        assert ms_max == 3.0
        assert total == 10.0e9
        assert s == 3.0
        assert gbps == pytest.approx(10.0e9 / 3.0e-3 / 1e9)


def test_single_rank_is_identity():
    import bench
    assert bench.rank_reduce(1.5, 1, None, "max") == 1.5
    gbps, ms, total = bench.replica_gbps(2.0e9, 4.0, 1, None)
    assert (ms, total) == (4.0, 2.0e9)
    assert gbps == pytest.approx(2.0e9 / 4.0e-3 / 1e9)
