"""Parity of the training step (moe_forward_train + moe_backward, through the C
ABI) with the float64 oracle's backward.

Every gradient -- dx, the router, expert and shared-expert weights, the shared
gate vector -- must satisfy max|g - g_ref| <= 1e-2 * max|g_ref| per tensor
(bf16 inputs and outputs, fp32 accumulation; the forward keeps its
pre-activations in bf16).  Routing is made unique by the margin rule of the
forward tests, so the GPU and the oracle differentiate the same selection.
Cases cover the tensor-core paths the backward takes: gathered and dense
operands, widths that are not multiples of the 64-wide K blocks (the gate/up
K split), experts without rows (zero gradients), renormalised and raw
softmax, sigmoid with a balance bias, the shared expert, one expert, single
tokens, layers large enough for the two-SM tiles (whole and partial), and the
full-size Gemma-upcycle layer.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_mixture_experts_sigmoid_b200 import binding as B
from sparse_mixture_experts_sigmoid_b200 import synth
from sparse_mixture_experts_sigmoid_b200.workloads import WORKLOADS, Workload

from support import OracleInputs, bits, enforce_margin, ocfg

pytestmark = pytest.mark.gpu

TOL = 1e-2
GRADS = ["dx", "dw_router", "dw_gate", "dw_up", "dw_down", "dsh_gate", "dsh_up", "dsh_down", "dw_shared_gate"]


def case(name, **kw):
    base = dict(T=300, d=256, E=16, h=384, k=4, seed=120, weight_std=0.05, router_std=0.05)
    base.update(kw)
    return Workload(name, **base)


CASES = [
    case("softmax_norm"),
    case("softmax_nonorm", norm_topk=False, seed=121),
    case("sigmoid_norm_shared", score="sigmoid", h_shared=192, seed=122),
    case("ragged_widths", d=200, h=136, seed=123),                # K blocks cut inside the gate/up split
    case("k1", k=1, seed=124),
    case("single_expert", E=1, k=1, seed=125),
    case("decode_T1", T=1, seed=126),
    case("few_tokens_shared", T=5, h_shared=64, seed=127),
    case("zipf_empty_experts", recipe="zipf", E=32, k=2, seed=128),
    case("many_experts", E=130, k=6, T=200, d=128, h=64, router_std=0.2, seed=129),
    # enough rows per expert (>= 512) and weight rows (>= 512) for the two-SM tiles
    case("pair_tiles", T=1024, d=512, E=4, h=512, k=2, seed=133),
    case("pair_ragged", T=800, d=576, E=3, h=640, k=2, seed=134),   # partial 256-row and 256-column tiles
]


def dy_for(w, device="cpu"):
    g = torch.Generator().manual_seed(w.seed + 7)
    return torch.randn(w.T, w.d, generator=g).to(torch.bfloat16).to(device)


def compare(grads, ref, names):
    for n in names:
        if n not in ref:
            continue
        got = grads[n].float().cpu().numpy().astype(np.float64)
        r = ref[n]
        scale = np.abs(r).max()
        err = np.abs(got - r).max()
        assert np.isfinite(got).all(), n
        if scale == 0:
            assert err == 0, n
            continue
        assert err <= TOL * scale, f"{n}: max|g - g_ref| = {err:.3e} > {TOL} * {scale:.3e}"


def run_case(w, bias=None):
    layer = synth.make_layer(w, "cpu")
    enforce_margin(w, layer, bias=bias)
    a = OracleInputs(layer)
    dev = layer.to("cuda")
    dy = dy_for(w)
    cfg = B.config_of(w)
    ws = B.alloc_train_workspace(cfg)
    bias_d = torch.from_numpy(bias).cuda() if bias is not None else None
    y = B.forward_train(cfg, dev, ws, balance_bias=bias_d)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    c = ocfg(w)
    y_ref = oracle.forward(c, a.x, a.wr, a.wg, a.wu, a.wd, a.shared, bias=bias)
    assert np.abs(y.float().cpu().numpy() - y_ref).max() <= TOL * np.abs(y_ref).max()
    grads = B.backward(cfg, dev, dy.cuda(), ws)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    ref = oracle.backward(c, a.x, a.wr, a.wg, a.wu, a.wd, bits(dy), a.shared, bias=bias)
    compare(grads, ref, GRADS)
    return grads, ref


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_backward_small(w):
    run_case(w)


def test_backward_with_balance_bias():
    w = case("sigmoid_bias", score="sigmoid", seed=130)
    b = (np.random.default_rng(131).standard_normal(w.E) * 0.05).astype(np.float32)
    run_case(w, bias=b)


def test_backward_zero_rows_expert_has_zero_gradient():
    """An expert that received no rows gets exactly zero weight gradients."""
    w = case("empty_expert", E=8, k=1, T=64, seed=132)
    layer = synth.make_layer(w, "cpu")
    layer.w_router[5] = -1.0          # with x = |x| + 0.1 expert 5 never wins
    layer.x[:, :] = layer.x.abs() + 0.1
    enforce_margin(w, layer)
    a = OracleInputs(layer)
    ids, _, _, _ = oracle.route(ocfg(w), a.x, a.wr)
    assert not (ids == 5).any()
    dev = layer.to("cuda")
    cfg = B.config_of(w)
    ws = B.alloc_train_workspace(cfg)
    B.forward_train(cfg, dev, ws)
    grads = B.backward(cfg, dev, dy_for(w, "cuda"), ws)
    torch.cuda.synchronize()
    for n in ("dw_gate", "dw_up", "dw_down"):
        assert grads[n][5].abs().max().item() == 0.0, n


def test_backward_full_size_gemma_upcycle():
    """The Gemma-upcycle layer at full size (2048 tokens, 256 experts of 32 rows on average)."""
    from test_gpu_parity import checked
    w = WORKLOADS["gemma_upcycle"]
    layer, dev, a = checked(w)
    dy = dy_for(w)
    cfg = B.config_of(w)
    ws = B.alloc_train_workspace(cfg)
    B.forward_train(cfg, dev, ws)
    grads = B.backward(cfg, dev, dy.cuda(), ws)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    ref = oracle.backward(ocfg(w), a.x, a.wr, a.wg, a.wu, a.wd, bits(dy), a.shared)
    compare(grads, ref, GRADS)


def test_backward_twice_is_reproducible_within_tolerance():
    """A second training step on the same workspace gives the same gradients up to
    the order of the fp32 additions into dx and the gate gradients."""
    w = CASES[0]
    g1, ref = run_case(w)
    layer = synth.make_layer(w, "cpu")
    enforce_margin(w, layer)
    dev = layer.to("cuda")
    cfg = B.config_of(w)
    ws = B.alloc_train_workspace(cfg)
    B.forward_train(cfg, dev, ws)
    g2 = B.backward(cfg, dev, dy_for(w, "cuda"), ws)
    torch.cuda.synchronize()
    compare(g2, ref, GRADS)
    # the weight gradients of the routed experts sum rows in grouped order: identical bits
    for n in ("dw_gate", "dw_up", "dw_down"):
        assert torch.equal(g1[n], g2[n]), n
