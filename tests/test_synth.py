"""The seeded input generator: determinism and the stated recipes."""
import math

import numpy as np
import torch

import oracle
from sparse_mixture_experts_sigmoid_b200 import synth
from sparse_mixture_experts_sigmoid_b200.workloads import WORKLOADS

from support import enforce_margin, ocfg, bits, MARGIN


def test_deterministic_and_independent():
    w = WORKLOADS["tiny"]
    a = synth.make_layer(w)
    b = synth.make_layer(w)
    for n in ("x", "w_router", "w_gate", "w_up", "w_down"):
        assert torch.equal(getattr(a, n), getattr(b, n))
    assert a.x.dtype == torch.float32
    # changing T keeps the weights
    c = synth.make_layer(w.with_(T=5))
    assert torch.equal(c.w_gate, a.w_gate) and c.x.shape == (5, w.d)


def test_upcycle_structure():
    w = WORKLOADS["gemma_upcycle"].with_(T=4, E=8, up_copies=4, up_slices=2, d=64, h=32)
    layer = synth.make_layer(w)
    wg = layer.w_gate.float()
    # copy 0 of each slice is the scaled slice; other copies differ in ~10% of entries
    for s in range(2):
        first = wg[s * 4]
        for c in range(1, 4):
            frac = (wg[s * 4 + c] != first).float().mean().item()
            assert 0.05 < frac < 0.15, frac
    # the two slices are different draws
    assert (wg[0] != wg[4]).float().mean().item() > 0.9
    # the scale: weights ~ N(0, (0.02*4)^2)
    assert abs(wg.std().item() - 0.08) < 0.01


def test_zipf_router_column():
    w = WORKLOADS["olmoe_zipf"].with_(T=16)
    layer = synth.make_layer(w)
    assert torch.all(layer.x[:, 0].float() == 1.0)
    col = layer.w_router[:, 0].float()
    # the column holds -a*ln(rank) for a permutation of ranks 1..E, rounded to bf16
    want = torch.tensor([-w.zipf_a * math.log(r) for r in range(1, w.E + 1)])
    got = torch.sort(col.double(), descending=True).values
    assert torch.allclose(got, want.double(), rtol=2 ** -8, atol=0)
    assert math.isclose(col.max().item(), 0.0, abs_tol=1e-6)


def test_margin_enforcement_and_redraw():
    w = WORKLOADS["gemma_upcycle"].with_(T=256)
    layer = synth.make_layer(w)
    before = layer.x.clone()
    n = enforce_margin(w, layer)
    m = oracle.topk_margin(ocfg(w), bits(layer.x), bits(layer.w_router))
    assert (m >= MARGIN).all()
    changed = (layer.x != before).any(dim=1).sum().item()
    assert changed <= n
    # redraw is keyed by (row, attempt): repeatable
    x2 = before.clone()
    synth.redraw_x_rows(w, x2, [3], 1)
    x3 = before.clone()
    synth.redraw_x_rows(w, x3, [3], 1)
    assert torch.equal(x2, x3) and not torch.equal(x2[3], before[3])
    assert torch.equal(x2[4], before[4])
    assert np.isfinite(m).all()
