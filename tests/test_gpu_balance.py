"""Parity of the load-balancing machinery with the float64 oracle, through the
C ABI:

* selection with a balance bias (moe_route_opts.balance_bias) on every router
  kernel (one CTA per token, the CUDA-core batched router in bf16 and fp32,
  the tensor-core router with 2..16 experts per lane): ids bit-exact, gates and
  scores within 1e-6, the layer output within 1e-2 * max|y_ref|;
* the score statistic P_e (moe_route_opts.score_mean) within 1e-6, and
  bit-identical from call to call;
* moe_update_bias bit-exact against the oracle's update (fp32 add), twice;
* moe_balance_loss against the oracle's Switch term.

"Small MoE Architecture, in depth", section "A small MoE layer in PyTorch"
and the auxiliary-loss-free balancing paragraph after it; "Mixture-of-Experts
-- more capacity per byte of weight", section "What's wired today".
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_mixture_experts_sigmoid_b200 import binding as B
from sparse_mixture_experts_sigmoid_b200 import synth
from sparse_mixture_experts_sigmoid_b200.workloads import WORKLOADS, Workload

from support import OracleInputs, enforce_margin, ocfg

pytestmark = pytest.mark.gpu

Y_TOL = 1e-2
GATE_TOL = 1e-6


def case(name, **kw):
    base = dict(T=300, d=256, E=16, h=384, k=4, score="sigmoid", seed=90)
    base.update(kw)
    return Workload(name, **base)


CASES = [
    case("sigmoid_norm_tc"),                                                   # tensor-core router
    case("softmax_nonorm_tc", score="softmax", norm_topk=False, seed=91),
    case("sigmoid_shared_tc", h_shared=256, seed=92),
    case("sigmoid_many_experts_tc", E=512, k=8, T=200, d=128, h=64, router_std=0.2, seed=93),
    case("sigmoid_130_experts_tc", E=130, k=6, T=160, d=128, h=64, router_std=0.2, seed=94),
    case("sigmoid_cuda_core_bf16", T=100, seed=95),                           # 64 < T < 128
    case("softmax_cuda_core_f32", score="softmax", dtype="f32", seed=96),
    case("sigmoid_cuda_core_f32_many", dtype="f32", E=80, k=5, T=150, d=128, h=64, router_std=0.2, seed=97),
    case("sigmoid_one_token_per_cta", T=40, seed=98),                         # T <= 64
    case("softmax_decode_T1", T=1, score="softmax", seed=99),
]


def _bias(w, seed):
    """A bias about the size of the score spread, so that it changes choices."""
    rng = np.random.default_rng(seed)
    spread = 0.05 if w.score == "sigmoid" else 0.5 / w.E
    return (rng.standard_normal(w.E) * spread).astype(np.float32)


_cache = {}


def layer_for(w):
    if w not in _cache:
        _cache.clear()
        b = _bias(w, w.seed + 1000)
        layer = synth.make_layer(w, "cpu")
        enforce_margin(w, layer, bias=b)
        _cache[w] = (layer, layer.to("cuda"), OracleInputs(layer), b)
    return _cache[w]


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_biased_route_and_score_mean(w):
    layer, dev, a, b = layer_for(w)
    c, cfg = ocfg(w), B.config_of(w)
    bias = torch.from_numpy(b).cuda()
    sm = torch.empty(w.E, dtype=torch.float32, device="cuda")
    ids, gates, probs, sg = B.route(cfg, dev.x, dev.w_router, dev.w_shared_gate, want_probs=True,
                                    balance_bias=bias, score_mean=sm)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    ids_ref, gates_ref, probs_ref, sg_ref = oracle.route(c, a.x, a.wr, a.w_sg, want_probs=True, bias=b)
    np.testing.assert_array_equal(ids.cpu().numpy(), ids_ref)
    np.testing.assert_allclose(gates.cpu().numpy(), gates_ref, rtol=0, atol=GATE_TOL)
    np.testing.assert_allclose(probs.cpu().numpy(), probs_ref, rtol=0, atol=GATE_TOL)
    if sg is not None:
        np.testing.assert_allclose(sg.cpu().numpy(), sg_ref, rtol=0, atol=GATE_TOL)
    ids_plain, _, _, _ = oracle.route(c, a.x, a.wr, a.w_sg)
    if w.T >= 40:
        assert (ids_plain != ids_ref).any(), "the bias should change some selections"
    P_ref = oracle.score_mean(c, a.x, a.wr)
    np.testing.assert_allclose(sm.cpu().numpy(), P_ref, rtol=0, atol=GATE_TOL)
    # the statistic is summed in a fixed order: identical bits on a second call
    sm2 = torch.empty_like(sm)
    B.route(cfg, dev.x, dev.w_router, dev.w_shared_gate, balance_bias=bias, score_mean=sm2)
    torch.cuda.synchronize()
    assert torch.equal(sm, sm2)


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_biased_forward_bias_update_and_switch_term(w):
    layer, dev, a, b = layer_for(w)
    c, cfg = ocfg(w), B.config_of(w)
    bias = torch.from_numpy(b).cuda()
    sm = torch.empty(w.E, dtype=torch.float32, device="cuda")
    ws = B.alloc_workspace(cfg)
    y = B.forward_layer(cfg, dev, ws=ws, balance_bias=bias, score_mean=sm)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    views = B.workspace_views(cfg, ws)
    ids_ref, gates_ref, _, _ = oracle.route(c, a.x, a.wr, a.w_sg, bias=b)
    np.testing.assert_array_equal(views["ids"].cpu().numpy(), ids_ref)
    np.testing.assert_allclose(views["gates"].cpu().numpy(), gates_ref, rtol=0, atol=GATE_TOL)
    counts_ref, _, _, _ = oracle.permute(c, ids_ref)
    np.testing.assert_array_equal(views["counts"].cpu().numpy(), counts_ref)
    y_ref = oracle.forward(c, a.x, a.wr, a.wg, a.wu, a.wd, a.shared, bias=b)
    yy = y.float().cpu().numpy()
    scale = np.abs(y_ref).max()
    assert np.abs(yy - y_ref).max() <= Y_TOL * scale
    P_ref = oracle.score_mean(c, a.x, a.wr)
    np.testing.assert_allclose(sm.cpu().numpy(), P_ref, rtol=0, atol=GATE_TOL)
    # the bias update from the step's counts, twice: bit-exact fp32
    lr = 1e-3
    ref = b.copy()
    for _ in range(2):
        B.update_bias(cfg, views["counts"], lr, bias)
        ref = oracle.update_bias(c, counts_ref, lr, ref)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(bias.cpu().numpy(), ref)
    # the Switch term from the same counts and the device's score means
    loss, frac = B.balance_loss(cfg, views["counts"], sm, 0.01, want_frac=True)
    torch.cuda.synchronize()
    loss_ref, f_ref = oracle.balance_loss(c, counts_ref, P_ref, 0.01)
    np.testing.assert_allclose(frac.cpu().numpy(), f_ref, rtol=1e-7, atol=0)
    np.testing.assert_allclose(loss.item(), loss_ref, rtol=1e-5)
    assert B.device_status() == 0


def test_score_mean_on_full_size_workloads():
    """P_e on the full-size workloads that the benchmark times (no bias), through
    moe_forward with the score statistic requested."""
    from test_gpu_parity import checked
    for name in ("gemma_upcycle", "olmoe_zipf", "qwen_shared", "mixtral_prefill", "mixtral_decode"):
        w = WORKLOADS[name]
        layer, dev, a = checked(w)
        cfg = B.config_of(w)
        sm = torch.empty(w.E, dtype=torch.float32, device="cuda")
        ws = B.alloc_workspace(cfg)
        B.forward_layer(cfg, dev, ws=ws, score_mean=sm)
        torch.cuda.synchronize()
        assert B.device_status() == 0
        P_ref = oracle.score_mean(ocfg(w), a.x, a.wr)
        np.testing.assert_allclose(sm.cpu().numpy(), P_ref, rtol=0, atol=GATE_TOL)
        counts = B.workspace_views(cfg, ws)["counts"]
        loss, _ = B.balance_loss(cfg, counts, sm, 0.01)
        loss_ref, _ = oracle.balance_loss(ocfg(w), counts.cpu().numpy(), P_ref, 0.01)
        np.testing.assert_allclose(loss.item(), loss_ref, rtol=1e-5)
        del ws


def test_balanced_load_keeps_the_bias():
    """counts exactly at the mean load leave the bias unchanged; one expert above
    it loses lr and the rest gain lr."""
    cfg = B.config(8, 64, 4, 64, 2)
    bias = torch.tensor([0.5, -0.25, 0.0, 1.0], dtype=torch.float32, device="cuda")
    B.update_bias(cfg, torch.tensor([4, 4, 4, 4], dtype=torch.int32, device="cuda"), 0.01, bias)
    torch.cuda.synchronize()
    assert bias.tolist() == [0.5, -0.25, 0.0, 1.0]
    B.update_bias(cfg, torch.tensor([7, 3, 3, 3], dtype=torch.int32, device="cuda"), 0.01, bias)
    torch.cuda.synchronize()
    f = np.float32
    assert bias.cpu().numpy().tolist() == [f(f(0.5) - f(0.01)), f(f(-0.25) + f(0.01)), f(0.01), f(f(1.0) + f(0.01))]
