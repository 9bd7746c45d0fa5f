"""Glue between the seeded input generator, the float64 oracle and the tests.

Only tests import this module.  It converts generator tensors into the stored
bits that the oracle reads, and it enforces the routing margin: every token's
top k+1 selection keys (computed by the oracle in float64 from the rounded
inputs) must be at least ``MARGIN`` apart, so that a correct fp32
implementation must select the same experts in the same slot order.  Rows
that fail are redrawn with the generator's per-row redraw, keyed by attempt.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from sparse_mixture_experts_sigmoid_b200 import synth
from sparse_mixture_experts_sigmoid_b200.workloads import Workload

MARGIN = 1e-3


def ocfg(w: Workload) -> oracle.Cfg:
    return oracle.Cfg(T=w.T, d=w.d, E=w.E, h=w.h, k=w.k, norm_topk=w.norm_topk, score=w.score,
                      h_shared=w.h_shared, dtype=w.dtype)


def bits(t: torch.Tensor | None):
    """CPU tensor -> numpy array of its stored bits (uint16 for bf16)."""
    if t is None:
        return None
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy()
    raise TypeError(t.dtype)


class OracleInputs:
    """Numpy views of one synthesised layer, in the oracle's argument order."""

    def __init__(self, layer: synth.Layer):
        self.x = bits(layer.x)
        self.wr = bits(layer.w_router)
        self.wg = bits(layer.w_gate)
        self.wu = bits(layer.w_up)
        self.wd = bits(layer.w_down)
        self.shared = None
        if layer.sh_gate is not None:
            self.shared = (bits(layer.sh_gate), bits(layer.sh_up), bits(layer.sh_down),
                           bits(layer.w_shared_gate))

    @property
    def w_sg(self):
        return None if self.shared is None else self.shared[3]


def enforce_margin(w: Workload, layer: synth.Layer, margin: float = MARGIN,
                   max_attempts: int = 80, bias=None) -> int:
    """Redraws x rows (in place, CPU tensor) until every token's selection margin
    (with the balance bias, when given) is >= margin.  Returns the number of row
    redraws."""
    c = ocfg(w)
    redraws = 0
    for attempt in range(1, max_attempts + 1):
        m = oracle.topk_margin(c, bits(layer.x), bits(layer.w_router), bias=bias)
        bad = np.nonzero(~(m >= margin))[0]
        if bad.size == 0:
            return redraws
        synth.redraw_x_rows(w, layer.x, bad, attempt)
        redraws += bad.size
    raise RuntimeError(f"margin not reached after {max_attempts} attempts for {w.name}")


def make_checked_layer(w: Workload) -> synth.Layer:
    """CPU layer with the routing margin enforced."""
    layer = synth.make_layer(w, "cpu")
    enforce_margin(w, layer)
    return layer
