"""Seeded synthetic inputs for a MoE layer workload.

This module draws random tensors and nothing else: it holds none of the
layer's arithmetic (no logits, scores, selection or expert math).  Every
tensor comes from its own ``torch.Generator`` seeded by a stable hash of
(workload seed, tensor name, index), so a tensor does not depend on which
other tensors were drawn, and any x row can be redrawn on its own.

Recipes (the distributions are those stated for each workload):

* ``normal`` -- x ~ N(0, x_std^2); router, expert and shared weights ~
  N(0, std^2).
* ``upcycle`` -- drop-upcycling ("Small models, sparse experts", section "How
  it works", step 2): one dense SwiGLU FFN of hidden width up_slices * h is
  drawn ~ N(0, weight_std^2) and split along its hidden dimension into
  ``up_slices`` slices; expert e is copy (e mod up_copies) of slice
  (e div up_copies); in every copy but the first, each weight is independently
  redrawn ~ N(0, weight_std^2) with probability ``up_redraw``; then every
  expert weight is multiplied by ``up_scale``.  Router ~ N(0, router_std^2).
* ``zipf`` -- as ``normal``, then feature 0 of every token is set to 1 and
  router column 0 is set to -zipf_a * ln(rank_e) for a seeded permutation of
  ranks 1..E, which skews expert loads towards a Zipf(zipf_a) spread.

Values are rounded once to the workload dtype (bf16 round-to-nearest-even, or
fp32 as drawn) before anything consumes them.
"""
from __future__ import annotations

import hashlib
import math
from dataclasses import dataclass

import torch

from .workloads import Workload


def _seed(*parts) -> int:
    h = hashlib.blake2b(repr(parts).encode(), digest_size=8).digest()
    return int.from_bytes(h, "little") & ((1 << 63) - 1)


def _gen(device, *parts) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_seed(*parts))
    return g


def _dtype(w: Workload):
    return torch.float32 if w.dtype == "f32" else torch.bfloat16


@dataclass
class Layer:
    """One layer's inputs.  Shapes: x[T,d], w_router[E,d], w_gate/w_up[E,h,d],
    w_down[E,d,h]; shared expert (or None): sh_gate/sh_up[h_s,d], sh_down[d,h_s],
    w_shared_gate[d]."""
    x: torch.Tensor
    w_router: torch.Tensor
    w_gate: torch.Tensor
    w_up: torch.Tensor
    w_down: torch.Tensor
    sh_gate: torch.Tensor | None = None
    sh_up: torch.Tensor | None = None
    sh_down: torch.Tensor | None = None
    w_shared_gate: torch.Tensor | None = None

    def to(self, device) -> "Layer":
        f = lambda t: None if t is None else t.to(device)
        return Layer(*(f(getattr(self, n)) for n in self.__dataclass_fields__))


def draw_x(w: Workload, device="cpu", T: int | None = None) -> torch.Tensor:
    """Token activations x[T, d] (attempt 0 for every row)."""
    T = w.T if T is None else T
    x = torch.randn(T, w.d, generator=_gen(device, w.seed, "x", 0), device=device) * w.x_std
    if w.recipe == "zipf":
        x[:, 0] = 1.0
    return x.to(_dtype(w))


def redraw_x_rows(w: Workload, x: torch.Tensor, rows, attempt: int) -> None:
    """Replaces rows of x in place by fresh draws keyed by (row, attempt >= 1)."""
    assert attempt >= 1
    for t in rows:
        t = int(t)
        r = torch.randn(w.d, generator=_gen("cpu", w.seed, "x-redraw", t, attempt)) * w.x_std
        if w.recipe == "zipf":
            r[0] = 1.0
        x[t] = r.to(_dtype(w)).to(x.device)


def _normal(device, shape, std, *parts):
    return torch.randn(*shape, generator=_gen(device, *parts), device=device) * std


def _experts_normal(w: Workload, device, name, rows, cols):
    dt = _dtype(w)
    out = torch.empty(w.E, rows, cols, dtype=dt, device=device)
    for e in range(w.E):
        out[e] = _normal(device, (rows, cols), w.weight_std, w.seed, name, e).to(dt)
    return out


def _experts_upcycle(w: Workload, device, name, rows, cols, hidden_axis):
    """Drop-upcycled expert stack; hidden_axis is 0 for gate/up [h, d], 1 for down [d, h]."""
    dt = _dtype(w)
    out = torch.empty(w.E, rows, cols, dtype=dt, device=device)
    base_shape = (rows * w.up_slices, cols) if hidden_axis == 0 else (rows, cols * w.up_slices)
    base = _normal(device, base_shape, w.weight_std, w.seed, name, "base")
    for e in range(w.E):
        s, c = divmod(e, w.up_copies)
        if hidden_axis == 0:
            sl = base[s * rows:(s + 1) * rows, :]
        else:
            sl = base[:, s * cols:(s + 1) * cols]
        sl = sl.clone()
        if c > 0:
            g = _gen(device, w.seed, name, "redraw", e)
            mask = torch.rand(rows, cols, generator=g, device=device) < w.up_redraw
            fresh = torch.randn(rows, cols, generator=g, device=device) * w.weight_std
            sl = torch.where(mask, fresh, sl)
        out[e] = (sl * w.up_scale).to(dt)
    return out


def make_layer(w: Workload, device="cpu") -> Layer:
    """Draws every input of workload ``w`` on ``device``.  The values depend on
    the device's generator: draw on the CPU when a CPU checker must see them."""
    dt = _dtype(w)
    x = draw_x(w, device)
    wr = _normal(device, (w.E, w.d), w.router_std, w.seed, "w_router")
    if w.recipe == "zipf":
        g = _gen("cpu", w.seed, "zipf-ranks")
        ranks = torch.randperm(w.E, generator=g).to(torch.float64) + 1.0
        col = torch.tensor([-w.zipf_a * math.log(r) for r in ranks.tolist()], dtype=torch.float32)
        wr[:, 0] = col.to(device)
    wr = wr.to(dt)
    if w.recipe == "upcycle":
        wg = _experts_upcycle(w, device, "w_gate", w.h, w.d, 0)
        wu = _experts_upcycle(w, device, "w_up", w.h, w.d, 0)
        wd = _experts_upcycle(w, device, "w_down", w.d, w.h, 1)
    else:
        wg = _experts_normal(w, device, "w_gate", w.h, w.d)
        wu = _experts_normal(w, device, "w_up", w.h, w.d)
        wd = _experts_normal(w, device, "w_down", w.d, w.h)
    layer = Layer(x, wr, wg, wu, wd)
    if w.h_shared:
        layer.sh_gate = _normal(device, (w.h_shared, w.d), w.weight_std, w.seed, "sh_gate").to(dt)
        layer.sh_up = _normal(device, (w.h_shared, w.d), w.weight_std, w.seed, "sh_up").to(dt)
        layer.sh_down = _normal(device, (w.d, w.h_shared), w.weight_std, w.seed, "sh_down").to(dt)
        layer.w_shared_gate = _normal(device, (w.d,), w.weight_std, w.seed, "w_s").to(dt)
    return layer
