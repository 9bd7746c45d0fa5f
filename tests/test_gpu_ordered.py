"""The ordered combine (moe_config.combine = MOE_COMBINE_ORDERED) through the
C ABI:

* the layer output against the float64 oracle, within the same tolerance as
  the default combine, on the tensor-core path (one-SM and two-SM tiles, with
  and without the shared expert, bf16 and fp32) and the small-batch path;
* bit-identical y over repeated calls (the point of the mode);
* moe_combine and moe_combine_noalloc in the ordered mode against the oracle,
  and bit-identical to each other;
* moe_forward_train's y bit-identical to moe_forward's in the ordered mode.

"Tutorial 11: Mixture of Experts (MoE)", section 3, Step 3 (unsort, then the
gate-weighted sum over the k experts): the sum is taken in slot order.
"""
import numpy as np
import pytest

import oracle
from sparse_mixture_experts_sigmoid_b200 import binding as B
from sparse_mixture_experts_sigmoid_b200.workloads import Workload

from support import OracleInputs, bits, make_checked_layer, ocfg

pytestmark = pytest.mark.gpu

Y_TOL = 1e-2


def case(name, **kw):
    base = dict(T=600, d=256, E=8, h=384, k=2, seed=140)
    base.update(kw)
    return Workload(name, **base)


CASES = [
    case("routed_bf16"),
    case("routed_pair_bf16", T=2048, d=512, E=4, h=512, k=2, seed=141),
    case("sigmoid_shared_bf16", score="sigmoid", h_shared=256, E=16, k=4, seed=142),
    case("f32_shared", dtype="f32", h_shared=128, T=300, seed=143),
    case("f32_routed", dtype="f32", T=300, seed=144),
    case("small_batch_T8", T=8, k=4, E=16, seed=145),
    case("decode_T1_shared", T=1, h_shared=256, seed=146),
]

_cache = {}


def layer_for(w):
    if w not in _cache:
        _cache.clear()
        layer = make_checked_layer(w)
        _cache[w] = (layer.to("cuda"), OracleInputs(layer))
    return _cache[w]


def _y_ref(w, a):
    return oracle.forward(ocfg(w), a.x, a.wr, a.wg, a.wu, a.wd, a.shared)


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_ordered_forward_matches_oracle_and_repeats_bit_for_bit(w):
    dev, a = layer_for(w)
    cfg = B.config_of(w, combine="ordered")
    ws = B.alloc_workspace(cfg)
    ys = []
    for _ in range(3):
        ys.append(B.forward_layer(cfg, dev, ws=ws).cpu())
        assert B.device_status() == 0
    y_ref = _y_ref(w, a)
    yy = ys[0].float().numpy().astype(np.float64)
    scale = np.abs(y_ref).max()
    assert np.abs(yy - y_ref).max() <= Y_TOL * scale
    for y in ys[1:]:
        assert np.array_equal(bits(y), bits(ys[0]))
    # the default combine gives the same result within the tolerance
    y_add = B.forward_layer(B.config_of(w), dev).cpu().float().numpy().astype(np.float64)
    assert np.abs(y_add - yy).max() <= Y_TOL * scale
    # the slot rows are exposed through the workspace views
    v = B.workspace_views(cfg, ws)
    assert v["y_slots"] is not None and tuple(v["y_slots"].shape) == (w.T * w.k, w.d)
    assert B.workspace_views(B.config_of(w), B.alloc_workspace(B.config_of(w)))["y_slots"] is None


COMBINE_CASES = [CASES[0], CASES[1], CASES[4], CASES[5]]


@pytest.mark.parametrize("w", COMBINE_CASES, ids=[w.name for w in COMBINE_CASES])
def test_ordered_combine_entry_points(w):
    dev, a = layer_for(w)
    c = ocfg(w)
    cfg = B.config_of(w, combine="ordered")
    ws = B.alloc_workspace(cfg)
    B.forward_layer(cfg, dev, ws=ws)
    v = B.workspace_views(cfg, ws)
    args = (v["act"], dev.w_down, v["offsets"], v["sorted_rows"], v["gates"])
    y1 = B.combine(cfg, *args).cpu()
    y2 = B.combine(cfg, *args).cpu()
    assert B.device_status() == 0
    assert np.array_equal(bits(y1), bits(y2))
    # oracle: the gate-weighted sum of the k expert rows (no shared expert here)
    assert w.h_shared == 0
    y_ref = oracle.forward(c, a.x, a.wr, a.wg, a.wu, a.wd, None)
    yy = y1.float().numpy().astype(np.float64)
    assert np.abs(yy - y_ref).max() <= Y_TOL * np.abs(y_ref).max()
    if w.T * w.k * w.d <= 4 << 20:
        y3 = B.combine_noalloc(cfg, *args).cpu()
        assert B.device_status() == 0
        assert np.array_equal(bits(y3), bits(y1))


TRAIN_CASES = [CASES[0], CASES[2]]


@pytest.mark.parametrize("w", TRAIN_CASES, ids=[w.name for w in TRAIN_CASES])
def test_ordered_forward_train_equals_forward(w):
    dev, _ = layer_for(w)
    cfg = B.config_of(w, combine="ordered")
    y_fwd = B.forward_layer(cfg, dev).cpu()
    ws = B.alloc_train_workspace(cfg)
    y_train = B.forward_train(cfg, dev, ws).cpu()
    assert B.device_status() == 0
    assert np.array_equal(bits(y_train), bits(y_fwd))
