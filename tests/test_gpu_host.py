"""moe_forward_host through the C ABI: x copied in from page-locked host
memory and y copied back by the call, in pieces whose copies overlap the
other pieces' layers.

* y against the float64 oracle (the layer of "Tutorial 11: Mixture of Experts
  (MoE)", section 4), for one and several pieces, with and without a copy
  stream, bf16 and fp32, with the shared expert;
* with the ordered combine, every piece's y bit-identical to moe_forward on
  that piece's tokens (the call is moe_forward per piece plus the copies);
* three or more pieces (the first and last half as large as the others),
  uneven splits, and more pieces than tokens.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_mixture_experts_sigmoid_b200 import binding as B
from sparse_mixture_experts_sigmoid_b200.workloads import Workload

from support import OracleInputs, bits, make_checked_layer, ocfg

pytestmark = pytest.mark.gpu

Y_TOL = 1e-2


def case(name, **kw):
    base = dict(T=600, d=256, E=8, h=384, k=2, seed=160)
    base.update(kw)
    return Workload(name, **base)


CASES = [
    case("routed_bf16"),
    case("routed_pair_bf16", T=2048, d=512, E=4, h=512, k=2, seed=161),
    case("sigmoid_shared_bf16", score="sigmoid", h_shared=256, E=16, k=4, seed=162),
    case("f32_shared", dtype="f32", h_shared=128, T=300, seed=163),
    case("decode_T5", T=5, E=16, k=4, seed=164),
]

_cache = {}


def layer_for(w):
    if w not in _cache:
        _cache.clear()
        layer = make_checked_layer(w)
        _cache[w] = (layer.to("cuda"), OracleInputs(layer))
    return _cache[w]


def host_pair(dev, w):
    xh = dev.x.cpu().pin_memory()
    yh = torch.full_like(xh, float("nan")).pin_memory()
    return xh, yh


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
@pytest.mark.parametrize("chunks,overlap", [(1, True), (2, False), (3, True), (4, True), (7, True)])
def test_forward_host_matches_oracle(w, chunks, overlap):
    dev, a = layer_for(w)
    cfg = B.config_of(w)
    xh, yh = host_pair(dev, w)
    cs = torch.cuda.Stream() if overlap else None
    B.forward_host(cfg, dev, xh, yh, chunks, copy_stream=cs)
    torch.cuda.current_stream().synchronize()
    assert B.device_status() == 0
    y_ref = oracle.forward(ocfg(w), a.x, a.wr, a.wg, a.wu, a.wd, a.shared)
    yy = yh.float().numpy().astype(np.float64)
    assert np.isfinite(yy).all()
    assert np.abs(yy - y_ref).max() <= Y_TOL * np.abs(y_ref).max()


@pytest.mark.parametrize("w", CASES[:3] + CASES[4:], ids=[w.name for w in CASES[:3] + CASES[4:]])
@pytest.mark.parametrize("chunks", [1, 3, 64])
def test_forward_host_pieces_equal_forward_on_their_tokens(w, chunks):
    dev, _ = layer_for(w)
    cfg = B.config_of(w, combine="ordered")
    xh, yh = host_pair(dev, w)
    ws = torch.empty(B.forward_host_workspace_size(cfg, chunks), dtype=torch.uint8, device="cuda")
    B.forward_host(cfg, dev, xh, yh, chunks, ws=ws, copy_stream=torch.cuda.Stream())
    torch.cuda.current_stream().synchronize()
    assert B.device_status() == 0
    b = B.host_piece_bounds(w.T, chunks)
    for t0, t1 in zip(b, b[1:]):
        if t1 == t0:
            continue
        pc = B.config_of(w, T=t1 - t0, combine="ordered")
        y = B.forward(pc, dev.x[t0:t1].contiguous(), dev.w_router, dev.w_gate, dev.w_up, dev.w_down,
                      dev.sh_gate, dev.sh_up, dev.sh_down, dev.w_shared_gate).cpu()
        assert np.array_equal(bits(y), bits(yh[t0:t1])), (t0, t1)
