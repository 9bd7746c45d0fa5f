"""The N > 1 host path of bench.py on CPU: two gloo ranks agree on the slowest
rank's step time and on the whole-job throughput (token-sharded replicas, so
no collective touches the data path; the only collectives are the barrier and
this max)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    ws, r, local = bench.dist_env()
    assert (ws, r, local) == (world, rank, rank)
    ms = bench.reduce_max(1.5 + rank, ws)          # rank 1 is the slow one
    val = bench.job_value(ws, 2048, ms)
    dist.barrier()
    dist.destroy_process_group()
    out[rank] = (ms, val)


def test_two_ranks_report_the_slowest_rank():
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0] == res[1]
    ms, val = res[0]
    assert ms == 2.5
    assert val == pytest.approx(2 * 2048 / 2.5e-3)


def test_single_process_is_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(3.0, 1) == 3.0
    assert bench.job_value(1, 100, 10.0) == pytest.approx(1e4)
