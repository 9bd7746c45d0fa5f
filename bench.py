#!/usr/bin/env python
"""MoE layer forward throughput on B200 (tokens/s), with the roofline of the
dominant kernel, an end-to-end figure through the public API with host
buffers, and the float64 oracle timed on the host cores as a baseline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One process per GPU (torchrun for N > 1).  Every rank runs the whole layer on
its own batch of T tokens (token-sharded replicas: the forward pass has no
exchange step, so there is no collective on the data path); the timed region
is bracketed by a barrier and a device synchronise, each step is timed with
CUDA events recorded by the library between its stages, and the slowest
rank's time is reported.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

from sparse_mixture_experts_sigmoid_b200 import binding as B
from sparse_mixture_experts_sigmoid_b200 import roofline, synth
from sparse_mixture_experts_sigmoid_b200.workloads import HEADLINE, WORKLOADS

ROOT = os.path.dirname(os.path.abspath(__file__))
METRIC = "MoE layer fwd tokens/s at 1 B200; % bf16 tensor peak (prefill) / % HBM BW (decode)"
L2_FLUSH_BYTES = 256 << 20   # twice the 126 MB L2
# stage -> (kernel name in the ncu launch list, source file whose hash keys the traffic figure)
GG_SRC = "grouped_gemm.cu+grouped_gemm2.cu"   # one-SM and two-SM grouped GEMM kernels
STAGE_KERNEL = {"route": ("router_logits_kernel", "router_tc.cu"), "permute": ("scatter_kernel", "permute.cu"),
                "gate_up": ("grouped_gemm_kernel", GG_SRC),
                "shared_gate_up": ("grouped_gemm_kernel", GG_SRC),
                "down": ("grouped_gemm_kernel", GG_SRC),
                "shared_down": ("grouped_gemm_kernel", GG_SRC),
                "finalize": ("finalize_kernel", "segment.cu")}
# kernels of the small-batch path (at most 64 assignments)
STAGE_KERNEL_SMALL = {"route": ("router_small_kernel", "router.cu"), "gate_up": ("seg_gateup_kernel", "segment.cu"),
                      "down": ("down_direct_kernel", "segment.cu")}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--workload", default=HEADLINE, choices=sorted(WORKLOADS))
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--cpu-seconds", type=float, default=15.0, help="budget of the oracle baseline sample")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    return p.parse_args()


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML on a thread."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.02):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period, self.index = period_s, index
        self._stop = threading.Event()
        self._t = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML missing: report no clocks rather than guess
            self.err = repr(e)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit and bit != 0x1:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------------------- helpers

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def reduce_max(v: float, ws: int) -> float:
    """Max over ranks (the slowest rank's time); identity on one process."""
    if ws == 1:
        return v
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_value(n_ranks: int, tokens_per_rank: int, ms_per_step: float) -> float:
    """Whole-job tokens/s: every rank processed its own batch in the slowest rank's step time."""
    return n_ranks * tokens_per_rank / (ms_per_step / 1e3)


def barrier(ws: int):
    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()


def source_hash(src: str) -> str:
    """Hash of a kernel's translation units ('+'-separated) plus the shared
    device headers."""
    d = os.path.join(ROOT, "sparse_mixture_experts_sigmoid_b200", "csrc")
    h = hashlib.sha256()
    for f in src.split("+") + sorted(x for x in os.listdir(d) if x.endswith(".cuh")):
        with open(os.path.join(d, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_for(stage: str, src: str, workload: str):
    """DRAM bytes per launch of a stage's kernel from a committed ncu capture
    (profiles/traffic.json), if the kernel's source is unchanged since."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            ent = json.load(f)[stage][workload]
        return float(ent["bytes_per_launch"]) if ent.get("src_sha") == source_hash(src) else None
    except (OSError, KeyError, ValueError):
        return None


def config_json(w, n):
    return {"workload": w.name, "T": w.T, "d": w.d, "E": w.E, "h": w.h, "k": w.k, "score": w.score,
            "norm_topk": w.norm_topk, "h_shared": w.h_shared, "global_batch_tokens": w.T * n,
            "parallelism": f"token-sharded replicas x{n} (no collective in the forward pass)",
            "l2": f"flushed between timed steps: write {L2_FLUSH_BYTES >> 20} MiB, then read another "
                  f"{L2_FLUSH_BYTES >> 20} MiB (no step input and no dirty line left in L2)"}


def dtype_name(w):
    return "f32" if w.dtype == "f32" else "bf16"


def _bits(t):
    if t is None:
        return None
    t = t.contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def run_oracle_sample(w, layer_cpu, seconds: float, max_tokens: int | None = None):
    """Times the float64 oracle on a sample of tokens sized to ~``seconds``.
    Returns (tokens, elapsed_s, threads, description)."""
    import oracle
    c = oracle.Cfg(T=w.T, d=w.d, E=w.E, h=w.h, k=w.k, norm_topk=w.norm_topk, score=w.score,
                   h_shared=w.h_shared, dtype=w.dtype)
    args = [_bits(layer_cpu.x), _bits(layer_cpu.w_router), _bits(layer_cpu.w_gate), _bits(layer_cpu.w_up),
            _bits(layer_cpu.w_down)]
    shared = None
    if w.h_shared:
        shared = (_bits(layer_cpu.sh_gate), _bits(layer_cpu.sh_up), _bits(layer_cpu.sh_down),
                  _bits(layer_cpu.w_shared_gate))
    nthreads = os.cpu_count() or 1
    rng = np.random.default_rng(7)
    # calibrate on one token per thread
    probe = rng.choice(w.T, size=min(w.T, nthreads), replace=False).astype(np.int64)
    t0 = time.perf_counter()
    oracle.forward(c, *args, shared, tokens=probe, nthreads=nthreads)
    per_tok = (time.perf_counter() - t0) / probe.size
    n = int(max(1, min(w.T, seconds / max(per_tok, 1e-9))))
    if max_tokens:
        n = min(n, max_tokens)
    tokens = np.sort(rng.choice(w.T, size=n, replace=False)).astype(np.int64)
    t0 = time.perf_counter()
    _, used = oracle.forward(c, *args, shared, tokens=tokens, nthreads=nthreads, return_threads=True)
    el = time.perf_counter() - t0
    return n, el, used, f"{n} of {w.T} tokens (seeded sample), all experts' math per token in float64"


# ----------------------------------------------------------------------------- arms

def bench_ours(args, w, ws_n, rank, local):
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    layer = synth.make_layer(w, dev)
    cfg = B.config_of(w)
    wsbuf = B.alloc_workspace(cfg, dev)
    y = torch.empty(w.T, w.d, dtype=layer.x.dtype, device=dev)
    flush_w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def flush():
        # evict everything: a write larger than L2, then a read of another buffer larger
        # than L2 so the write's dirty lines are written back before the step, not during it
        flush_w.zero_()
        flush_r.sum()

    K, W = args.steps, args.warmup

    for _ in range(W):
        B.forward_layer(cfg, layer, y=y, ws=wsbuf)
    torch.cuda.synchronize()
    counts = B.workspace_views(cfg, wsbuf)["counts"].cpu().numpy()

    # timed region: K steps, each bracketed by CUDA events on the launching stream
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    stops = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    sampler = ClockSampler(local)
    with sampler:
        barrier(ws_n)
        l0 = B.launch_count()
        for i in range(K):
            flush()
            starts[i].record()
            B.forward_layer(cfg, layer, y=y, ws=wsbuf)
            stops[i].record()
        barrier(ws_n)
        launches = B.launch_count() - l0
    assert B.device_status() == 0, "device error flag set during the timed region"
    step_ms = [a.elapsed_time(b) for a, b in zip(starts, stops)]
    ms_local = statistics.fmean(step_ms)
    ms = reduce_max(ms_local, ws_n)
    value = job_value(ws_n, w.T, ms)

    # per-kernel breakdown: the same steps again with the library recording an
    # event after each stage (the dominant kernel's roofline comes from these)
    ev = [B.StageEvents() for _ in range(K)]
    barrier(ws_n)
    for i in range(K):
        flush()
        with ev[i]:
            B.forward_layer(cfg, layer, y=y, ws=wsbuf)
    barrier(ws_n)
    stage = {n: statistics.fmean(e.stage_ms()[n] for e in ev) for n in B.STAGES}

    # end to end through the public API: pinned host x in, y back to pinned host
    e2e = None
    if not args.no_e2e:
        xh = layer.x.cpu().pin_memory()
        yh = torch.empty(w.T, w.d, dtype=y.dtype).pin_memory()
        xd = torch.empty_like(layer.x)
        e2e_layer = synth.Layer(xd, layer.w_router, layer.w_gate, layer.w_up, layer.w_down, layer.sh_gate,
                                layer.sh_up, layer.sh_down, layer.w_shared_gate)
        for _ in range(3):
            xd.copy_(xh, non_blocking=True)
            B.forward_layer(cfg, e2e_layer, y=y, ws=wsbuf)
            yh.copy_(y, non_blocking=True)
        barrier(ws_n)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        tot = 0.0
        for _ in range(K):
            flush()
            s0.record()
            xd.copy_(xh, non_blocking=True)
            B.forward_layer(cfg, e2e_layer, y=y, ws=wsbuf)
            yh.copy_(y, non_blocking=True)
            s1.record()
            s1.synchronize()
            tot += s0.elapsed_time(s1)
        barrier(ws_n)
        e2e_ms = reduce_max(tot / K, ws_n)
        e2e = {"value": job_value(ws_n, w.T, e2e_ms), "unit": "tokens/s", "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": xh.numel() * xh.element_size(),
               "d2h_bytes_per_step": yh.numel() * yh.element_size()}

    # roofline of the dominant kernel
    peaks = roofline.measured_peaks()
    work = roofline.stage_work(w, counts)
    dom = max((n for n in stage if n in work), key=lambda n: stage[n])
    fl, by = work[dom]["flops"], work[dom]["bytes"]
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    t = stage[dom] / 1e3
    kname, ksrc = STAGE_KERNEL[dom]
    if w.R <= B.decode_max_rows() and dom in STAGE_KERNEL_SMALL:
        kname, ksrc = STAGE_KERNEL_SMALL[dom]
    if by > 0 and fl / by < ridge:
        roof = {"bound": "hbm", "achieved": by / t / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": fl / t / 1e12, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = traffic_for(dom, ksrc, w.name)
    roof.update({"kernel": kname, "stage": dom, "ms_per_launch": stage[dom],
                 "algorithmic_bytes": by, "algorithmic_flops": fl, "peak_source": peaks["source"]})
    lw = roofline.layer_work(w, counts)
    layer_roof = {"tflops": lw["flops"] / (ms / 1e3) / 1e12, "gbs": lw["bytes"] / (ms / 1e3) / 1e9,
                  "tensor_frac": lw["flops"] / (ms / 1e3) / 1e12 / peaks["bf16_tflops"],
                  "hbm_frac": lw["bytes"] / (ms / 1e3) / 1e9 / peaks["hbm_gbs"]}

    out = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws_n, "steps": K, "warmup": W,
           "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
           "dtype": dtype_name(w), "data": "synthetic (seeded; shapes and distributions of the workload)",
           "config": config_json(w, ws_n), "roofline": roof, "layer_roofline": layer_roof,
           "stages_ms": stage, "gpu_launches": launches, "clocks": sampler.summary(), "e2e": e2e,
           "active_experts": int(np.count_nonzero(counts))}

    if rank == 0 and ws_n == 1 and not args.no_cpu_baseline:
        layer_cpu = layer.to("cpu")
        n, el, used, desc = run_oracle_sample(w, layer_cpu, args.cpu_seconds)
        out["cpu_baseline"] = {"value": n / el, "unit": "tokens/s", "cores": used, "kind": "oracle",
                               "sample": desc, "seconds": el}
    return out


def bench_reference(args, w, ws_n, rank):
    """The oracle as the reference arm: each step is a bounded sample of the workload."""
    if rank != 0:
        return None
    layer_cpu = synth.make_layer(w, "cpu")
    K, W = args.steps, args.warmup
    per_step = max(0.05, 150.0 / max(1, K + W))
    import oracle
    c = oracle.Cfg(T=w.T, d=w.d, E=w.E, h=w.h, k=w.k, norm_topk=w.norm_topk, score=w.score,
                   h_shared=w.h_shared, dtype=w.dtype)
    args_ = [_bits(layer_cpu.x), _bits(layer_cpu.w_router), _bits(layer_cpu.w_gate), _bits(layer_cpu.w_up),
             _bits(layer_cpu.w_down)]
    shared = None
    if w.h_shared:
        shared = (_bits(layer_cpu.sh_gate), _bits(layer_cpu.sh_up), _bits(layer_cpu.sh_down),
                  _bits(layer_cpu.w_shared_gate))
    nthreads = os.cpu_count() or 1
    rng = np.random.default_rng(11)
    probe = rng.choice(w.T, size=min(w.T, nthreads), replace=False).astype(np.int64)
    t0 = time.perf_counter()
    oracle.forward(c, *args_, shared, tokens=probe, nthreads=nthreads)
    per_tok = (time.perf_counter() - t0) / probe.size
    n = int(max(1, min(w.T, per_step / max(per_tok, 1e-9))))
    used = nthreads
    tot_tok, tot_s = 0, 0.0
    for i in range(W + K):
        toks = np.sort(rng.choice(w.T, size=n, replace=False)).astype(np.int64)
        t0 = time.perf_counter()
        _, used = oracle.forward(c, *args_, shared, tokens=toks, nthreads=nthreads, return_threads=True)
        el = time.perf_counter() - t0
        if i >= W:
            tot_tok += n
            tot_s += el
    value = tot_tok / tot_s
    desc = f"{n} of {w.T} tokens per step (seeded samples), float64 per-token oracle"
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws_n,
            "steps": K, "warmup": W, "ms_per_step": tot_s / K * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
            "config": config_json(w, ws_n),
            "cpu_baseline": {"kind": "oracle", "cores": used, "sample": desc, "value": value, "unit": "tokens/s"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    ws_n, rank, local = dist_env()
    if ws_n != args.gpus and not (ws_n == 1 and args.gpus == 1):
        if ws_n == 1:
            sys.exit(f"--gpus {args.gpus} needs one process per GPU: launch with torchrun")
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        out = bench_reference(args, w, ws_n, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    if ws_n > 1:
        from datetime import timedelta
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    try:
        out = bench_ours(args, w, ws_n, rank, local)
    finally:
        if ws_n > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
