"""bench.py's multi-rank path on CPU: two gloo ranks, each timing a different
interval; both must report the maximum, and the whole-job throughput counts
every rank's units over that maximum (weak scaling, no data-path collective)."""

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


def _rank(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    ms = [12.5, 20.0][rank]
    m = bench.max_over_ranks(ms)
    out[rank] = (m, bench.job_throughput(32760, 10, world, m))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_and_job_throughput():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0] == res[1]
    m, v = res[0]
    assert m == 20.0
    assert v == pytest.approx(2 * 32760 * 10 / 0.020)


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_throughput(100, 4, 1, 2.0) == pytest.approx(100 * 4 / 0.002)
