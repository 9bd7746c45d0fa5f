"""Roofline arithmetic for the benchmark: algorithmic work per kernel and the
bandwidth ceiling of batch-1 decode.

Algorithmic counts exclude padding and tile waste.  Bytes count what a kernel
must move at least once: the weights of the experts that received rows, its
inputs and its outputs.
"""
from __future__ import annotations

import json
import os

import numpy as np

from .workloads import Workload

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def batch1_decode_ceiling(total_params: float, active_params: float, bytes_per_param: float,
                          mem_gb_s: float) -> tuple[float, float]:
    """(memory footprint in GB, upper bound on decode tokens/s): every active
    weight is read once per token ("Small MoE Architecture, in depth", section
    "Worked example: the batch-1 budget on a device")."""
    footprint_gb = total_params * bytes_per_param / 1e9
    per_token_gb = active_params * bytes_per_param / 1e9
    return footprint_gb, mem_gb_s / per_token_gb


def active_experts(counts) -> int:
    return int(np.count_nonzero(np.asarray(counts)))


# 4-bit routed expert weights: half a byte per parameter plus one fp32 scale per 64
Q4_BYTES_PER_PARAM = 0.5 + 4.0 / 64


def stage_work(w: Workload, counts, q4: bool = False) -> dict:
    """Algorithmic FLOPs and bytes of each stage of the forward pass, given the
    per-expert row counts the router produced (q4: routed experts in 4 bits)."""
    esz = w.elem_bytes()
    wsz = Q4_BYTES_PER_PARAM if q4 else esz   # bytes per routed expert parameter
    R, T, d, h, hs = w.R, w.T, w.d, w.h, w.h_shared
    na = active_experts(counts)
    work = {
        "route": {"flops": 2.0 * T * w.E * d + (2.0 * T * d if hs else 0.0),
                  "bytes": T * d * esz + w.E * d * esz + R * 8 + (d * esz + T * 4 if hs else 0)},
        "permute": {"flops": 0.0, "bytes": R * 4 * 3 + (2 * w.E + 1) * 4},
        "gate_up": {"flops": 2.0 * R * 2 * h * d,
                    "bytes": na * 2 * h * d * wsz + T * d * esz + R * h * esz},
        "down": {"flops": 2.0 * R * h * d,
                 "bytes": na * d * h * wsz + R * h * esz + R * 8 + T * d * 4},
        "finalize": {"flops": 0.0, "bytes": T * d * (4 + esz) if w.dtype == "bf16" else 0},
    }
    if hs:
        work["shared_gate_up"] = {"flops": 2.0 * T * 2 * hs * d, "bytes": 2 * hs * d * esz + T * d * esz
                                  + T * hs * esz}
        work["shared_down"] = {"flops": 2.0 * T * hs * d, "bytes": d * hs * esz + T * hs * esz + T * 4
                               + T * d * 4}
    return work


def layer_work(w: Workload, counts, q4: bool = False) -> dict:
    """Whole-layer algorithmic FLOPs and minimum bytes (weights of the chosen
    experts, router, x and y; q4: routed experts in 4 bits)."""
    esz = w.elem_bytes()
    na = active_experts(counts)
    wsz = Q4_BYTES_PER_PARAM if q4 else esz
    b = na * 3 * w.h * w.d * wsz + w.E * w.d * esz + 2 * w.T * w.d * esz
    if w.h_shared:
        b += 3 * w.h_shared * w.d * esz + w.d * esz
    return {"flops": w.flops(), "bytes": b}


def measured_peaks(path: str | None = None) -> dict:
    """The measured peaks (MEASURED_PEAKS.json), else the machine's fallback figures."""
    path = path or os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


def load_spread(counts) -> dict:
    """The realised per-expert load: rows per expert (max, min, mean), their
    coefficient of variation, and how many experts received rows."""
    c = np.asarray(counts, dtype=np.float64)
    mean = float(c.mean()) if c.size else 0.0
    return {"active_experts": int(np.count_nonzero(c)), "max": int(c.max()) if c.size else 0,
            "min": int(c.min()) if c.size else 0, "mean": mean,
            "cv": float(c.std() / mean) if mean > 0 else 0.0}


def fractions(flops: float, nbytes: float, seconds: float, peaks: dict, tensor_peak: float) -> dict:
    """Both roofline fractions of one timed piece of work and the binding one.

    tensor_frac = (flops / t) / tensor_peak and hbm_frac = (bytes / t) / HBM
    peak; the roofline's lower bound on the time is max(flops / tensor_peak,
    bytes / HBM peak), so frac = that bound / t = max(tensor_frac, hbm_frac),
    and `bound` names the resource that sets it."""
    tf = flops / seconds / 1e12 / tensor_peak if seconds > 0 else 0.0
    hf = nbytes / seconds / 1e9 / peaks["hbm_gbs"] if seconds > 0 else 0.0
    bound = "tensor" if tf >= hf else "hbm"
    return {"bound": bound, "tensor_frac": tf, "hbm_frac": hf, "frac": max(tf, hf),
            "tflops": flops / seconds / 1e12 if seconds > 0 else 0.0,
            "gbs": nbytes / seconds / 1e9 if seconds > 0 else 0.0}
