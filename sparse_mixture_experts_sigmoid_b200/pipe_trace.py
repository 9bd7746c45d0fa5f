"""Pipeline trace of the grouped GEMM kernels: a diagnostic build, not the product.

``-DMOE_PIPE_TRACE`` compiles clock counters into the tcgen05 GEMM kernels (the
forward's one-SM and two-SM kernels and the backward's): per kernel variant,
SM cycles summed over CTAs for the whole kernel, the MMA issuer waiting for
operands and for a free accumulator, the producers waiting for a free ring
stage, epilogue warp 0 waiting for an accumulator and draining one, and the
first gather thread waiting for a stage.  This module builds that variant as
``libmoe_trace.so`` next to ``libmoe.so`` (objects under ``_build/trace``) and
prints the shares for a few steps of the named workloads::

    python -m sparse_mixture_experts_sigmoid_b200.pipe_trace --build
    python -m sparse_mixture_experts_sigmoid_b200.pipe_trace --backward olmoe_zipf mixtral_prefill
    python -m sparse_mixture_experts_sigmoid_b200.pipe_trace --forward olmoe_zipf

Times are SM cycles per CTA divided by the 1965 MHz maximum clock (so they
understate wall time when the clock ran lower).  In a two-SM kernel only the
even CTA issues MMAs: its waits are shares of that CTA's time.
"""
from __future__ import annotations

import ctypes
import glob
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

from . import build as _build

TRACE_LIB = os.path.join(_build.PKG, "libmoe_trace.so")
_MHZ = 1965.0


def build_trace() -> str:
    out = os.path.join(_build.BUILD, "trace")
    os.makedirs(out, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(_build.CSRC, "*.cu")))
    objs = [os.path.join(out, os.path.basename(s)[:-3] + ".o") for s in srcs]

    def run(cmd):
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode:
            raise RuntimeError(" ".join(cmd) + "\n" + r.stdout + r.stderr)

    jobs = [[_build.nvcc(), *_build.ARCH, *_build.NVCC_FLAGS, "-DMOE_PIPE_TRACE", "-c", s, "-o", o]
            for s, o in zip(srcs, objs)]
    with ThreadPoolExecutor(max_workers=max(1, min(len(jobs), os.cpu_count() or 4))) as ex:
        list(ex.map(run, jobs))
    run([_build.nvcc(), *_build.ARCH, "-shared", "-Xcompiler", "-fPIC", "-o", TRACE_LIB, *objs])
    return TRACE_LIB


def _lib():
    from . import binding as B
    if not os.path.exists(TRACE_LIB):
        raise RuntimeError(f"{TRACE_LIB} is missing: run with --build first")
    B.LIB_PATH = TRACE_LIB
    L = B.lib()
    for name in ("moe_debug_pipe_trace", "moe_debug_fwd_trace", "moe_debug_fwd2_trace"):
        getattr(L, name).argtypes = [ctypes.c_void_p, ctypes.c_int]
    return B, L


def _read(fn):
    buf = (ctypes.c_ulonglong * 64)()
    if fn(buf, 1) != 0:
        raise RuntimeError("reading the trace counters failed")
    return [list(buf[8 * i:8 * i + 8]) for i in range(8)]


def _row(name, v, pair):
    tot, full, tempty, empty, tfull, body, n, gwait = v
    if n == 0 or tot == 0:
        return None
    mma = 2.0 if pair else 1.0   # the even CTA's MMA waits over that CTA's time
    return (f"  {name:22s} CTAs {n:5d} | per CTA {tot / n / _MHZ:8.1f} us | MMA waits operands "
            f"{100 * mma * full / tot:5.1f}% accumulator {100 * mma * tempty / tot:5.1f}% | producers wait "
            f"{100 * empty / tot:5.1f}% | gather waits {100 * gwait / tot:5.1f}% | epilogue waits "
            f"{100 * tfull / tot:5.1f}% drains {100 * body / tot:5.1f}%")


def _print(rows):
    for r in rows:
        if r:
            print(r)


def main(argv: list[str]) -> int:
    if "--build" in argv:
        print(build_trace())
        argv = [a for a in argv if a != "--build"]
        if not argv:
            return 0
    backward = "--backward" in argv
    names = [a for a in argv if not a.startswith("--")]
    import torch
    B, L = _lib()
    from . import synth
    from .workloads import WORKLOADS
    for wn in names:
        w = WORKLOADS[wn]
        layer = synth.make_layer(w, "cuda")
        cfg = B.config_of(w)
        print(wn)
        if backward:
            ws = B.alloc_train_workspace(cfg)
            dy = torch.randn(w.T, w.d, device="cuda").to(layer.x.dtype)
            for i in range(3):
                B.forward_train(cfg, layer, ws)
                if i == 2:
                    _read(L.moe_debug_pipe_trace)   # count the last backward only
                B.backward(cfg, layer, dy, ws)
            torch.cuda.synchronize()
            v = _read(L.moe_debug_pipe_trace)
            kinds = ["SwiGLU", "scatter", "weight gradients"]
            _print([_row(f"{kinds[i]} (one SM)", v[i], False) for i in range(3)] +
                    [_row(f"{kinds[i - 4]} (two SMs)", v[i], True) for i in range(4, 7)])
            del ws
        else:
            for tag, train in (("forward", False), ("training forward", True)):
                ws = B.alloc_train_workspace(cfg) if train else B.alloc_workspace(cfg)
                for i in range(4):
                    if i == 3:
                        _read(L.moe_debug_fwd_trace)
                        _read(L.moe_debug_fwd2_trace)
                    if train:
                        B.forward_train(cfg, layer, ws)
                    else:
                        B.forward_layer(cfg, layer, ws=ws)
                torch.cuda.synchronize()
                one, two = _read(L.moe_debug_fwd_trace), _read(L.moe_debug_fwd2_trace)
                print(f" {tag}")
                _print([_row(f"{k} (one SM)", one[i], False) for i, k in enumerate(["gate/up", "down", "down, 64 rows"])] +
                       [_row(f"{k} (two SMs)", two[i], True) for i, k in
                        enumerate(["gate/up, gathered", "gate/up, dense", "down"])])
                del ws
        del layer
        torch.cuda.empty_cache()
    return 0


if __name__ == "__main__":
    sys.exit(main(sys.argv[1:]))
