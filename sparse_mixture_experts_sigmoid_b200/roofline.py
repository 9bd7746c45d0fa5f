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


def stage_work(w: Workload, counts) -> dict:
    """Algorithmic FLOPs and bytes of each stage of the forward pass, given the
    per-expert row counts the router produced."""
    esz = w.elem_bytes()
    R, T, d, h, hs = w.R, w.T, w.d, w.h, w.h_shared
    na = active_experts(counts)
    work = {
        "route": {"flops": 2.0 * T * w.E * d + (2.0 * T * d if hs else 0.0),
                  "bytes": T * d * esz + w.E * d * esz + R * 8 + (d * esz + T * 4 if hs else 0)},
        "permute": {"flops": 0.0, "bytes": R * 4 * 3 + (2 * w.E + 1) * 4},
        "gate_up": {"flops": 2.0 * R * 2 * h * d,
                    "bytes": na * 2 * h * d * esz + T * d * esz + R * h * esz},
        "down": {"flops": 2.0 * R * h * d,
                 "bytes": na * d * h * esz + R * h * esz + R * 8 + T * d * 4},
        "finalize": {"flops": 0.0, "bytes": T * d * (4 + esz) if w.dtype == "bf16" else 0},
    }
    if hs:
        work["shared_gate_up"] = {"flops": 2.0 * T * 2 * hs * d, "bytes": 2 * hs * d * esz + T * d * esz
                                  + T * hs * esz}
        work["shared_down"] = {"flops": 2.0 * T * hs * d, "bytes": d * hs * esz + T * hs * esz + T * 4
                               + T * d * 4}
    return work


def layer_work(w: Workload, counts) -> dict:
    """Whole-layer algorithmic FLOPs and minimum bytes (weights of the chosen
    experts, router, x and y)."""
    esz = w.elem_bytes()
    na = active_experts(counts)
    b = na * 3 * w.h * w.d * esz + w.E * w.d * esz + 2 * w.T * w.d * esz
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
