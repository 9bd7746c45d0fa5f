"""The N > 1 host path on CPU, as gloo ranks:

* bench.py: two ranks agree on the slowest rank's step time and on the
  whole-job throughput (token-sharded replicas, so no collective touches the
  data path; the only collectives are the barrier and this max);
* the library's host path per rank: each rank validates its own shard of the
  tokens, sizes and carves its workspace (forward and training), and is
  refused the same bad arguments, and the ranks' results agree with each other
  and with the shard arithmetic."""
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


def _worker_host_path(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import ctypes
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    from sparse_mixture_experts_sigmoid_b200 import binding as B
    from sparse_mixture_experts_sigmoid_b200.workloads import WORKLOADS
    res = {}
    for name in ("gemma_upcycle", "olmoe_zipf", "qwen_shared", "mixtral_prefill"):
        w = WORKLOADS[name]
        # token-sharded replicas: every rank holds all experts and its own T tokens
        cfg = B.config_of(w)
        assert B.validate(cfg) == 0
        n = B.workspace_size(cfg)
        nt = B.train_workspace_size(cfg)
        v = B.WorkspaceViews()
        base = (1 << 40) + rank * (1 << 36)          # distinct fake device ranges per rank
        assert B.lib().moe_workspace_layout(ctypes.byref(cfg), ctypes.c_void_p(base), n, ctypes.byref(v)) == 0
        offs = [getattr(v, f) - base if getattr(v, f) else -1 for f, _ in B.WorkspaceViews._fields_]
        # an undersized workspace is refused before anything is launched, on every rank
        fake = ctypes.c_void_p(0x1000)
        args = [fake] * 5 + ([fake] * 4 if w.h_shared else [None] * 4) + [fake]
        assert B.lib().moe_forward(ctypes.byref(cfg), None, *args, ctypes.c_void_p(base), n - 256, None) == 3
        t = torch.tensor([n, nt] + offs, dtype=torch.int64)
        gathered = [torch.zeros_like(t) for _ in range(world)]
        dist.all_gather(gathered, t)
        res[name] = [g.tolist() for g in gathered]
    dist.barrier()
    dist.destroy_process_group()
    out[rank] = res


def test_each_rank_runs_the_host_path_for_its_shard():
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_worker_host_path, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(180)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0] == res[1]
    for name, (r0, r1) in res[0].items():
        # same shard shape on both ranks: identical sizes and layouts
        assert r0 == r1, name
        n, nt = r0[0], r0[1]
        assert nt > n > 0, name
