"""Parity of the 4-bit routed experts (moe_quantize_q4, moe_forward_q4, through
the C ABI) with the float64 oracle.

* The codes and scales are bit-exact with the oracle's quantiser (integer
  work; the code is decided in fp32 on both sides).
* The layer on the represented weights: routing bit-exact, output within
  max|y - y_ref| <= 1e-2 * max|y_ref| (the oracle dequantises the codes and
  runs its float64 forward).
* The full-size Mixtral-like batch-1 decode step, checked against the
  oracle's routing and the dense SwiGLU of the two chosen experts on their
  dequantised weights.
"Small MoE Architecture, in depth", "Worked example: the batch-1 budget on a
device" and "Running experts that do not fit: offloading and quantisation".
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import dense
from sparse_mixture_experts_sigmoid_b200 import binding as B
from sparse_mixture_experts_sigmoid_b200 import synth
from sparse_mixture_experts_sigmoid_b200.workloads import WORKLOADS, Workload

from support import OracleInputs, bits, enforce_margin, make_checked_layer, ocfg

pytestmark = pytest.mark.gpu

TOL = 1e-2


def test_quantize_bit_exact_with_the_oracle():
    g = torch.Generator().manual_seed(5)
    for dt in (torch.bfloat16, torch.float32):
        w = (torch.randn(37, 320, generator=g) * torch.rand(37, 1, generator=g) * 3).to(dt)
        w[3, 64:128] = 0                       # an all-zero group
        w[5, :64] = torch.linspace(-3.5, 3.5, 64).to(dt)
        q, sc = B.quantize_q4(w.cuda())
        torch.cuda.synchronize()
        q_ref, sc_ref = oracle.quantize_q4(bits(w))
        np.testing.assert_array_equal(q.cpu().numpy(), q_ref)
        np.testing.assert_array_equal(sc.cpu().numpy(), sc_ref)


def case(name, **kw):
    base = dict(T=1, d=512, E=16, h=384, k=4, seed=140)
    base.update(kw)
    return Workload(name, **base)


CASES = [
    case("decode_T1"),
    case("decode_T1_shared", h_shared=256, seed=141),
    case("decode_T3_k8", T=3, E=64, k=8, d=256, h=128, router_std=0.2, seed=142),
    case("decode_T16_k4", T=16, seed=143),
    case("decode_sigmoid_nonorm", score="sigmoid", norm_topk=False, T=2, seed=144),
    # d and h multiples of 256: the kernels that stream the codes through a
    # shared-memory ring (a last partial 1024-element chunk in the second and
    # third; experts holding more than two rows, so several passes, in the others)
    case("ring_decode_T1", h=512, seed=145),
    case("ring_T16_shared_ragged_chunks", T=16, d=768, h=1280, h_shared=256, seed=146),
    case("ring_T16_E4_k1", T=16, E=4, k=1, d=256, h=1280, seed=147),
    case("ring_T3_k8", T=3, E=64, k=8, d=256, h=256, router_std=0.2, seed=148),
]


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_forward_q4_small(w):
    layer = make_checked_layer(w)
    a = OracleInputs(layer)
    dev = layer.to("cuda")
    cfg = B.config_of(w)
    q4 = B.quantize_experts_q4(dev)
    ws = B.alloc_workspace(cfg)
    y = B.forward_q4(cfg, dev, q4, ws=ws)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    views = B.workspace_views(cfg, ws)
    ids_ref, _, _, _ = oracle.route(ocfg(w), a.x, a.wr, a.w_sg)
    np.testing.assert_array_equal(views["ids"].cpu().numpy(), ids_ref)
    qs = [(q4["q_" + n].cpu().numpy(), q4["s_" + n].cpu().numpy()) for n in ("gate", "up", "down")]
    y_ref = oracle.forward_q4(ocfg(w), a.x, a.wr, *qs[0], *qs[1], *qs[2], a.shared)
    err = np.abs(y.float().cpu().numpy() - y_ref).max()
    assert err <= TOL * np.abs(y_ref).max(), err


def test_forward_q4_rejects_batches_beyond_the_decode_path():
    w = case("big", T=100)
    cfg = B.config_of(w)
    import ctypes
    fake = ctypes.c_void_p(0x1000)
    st = B.lib().moe_forward_q4(ctypes.byref(cfg), None, *([fake] * 8), None, None, None, None, fake,
                                ctypes.c_void_p(1 << 20), 1 << 30, None)
    assert st == 2          # MOE_ERR_UNSUPPORTED


def test_forward_q4_full_size_mixtral_decode():
    """One token through the Mixtral-like layer (8 experts of 4096 x 14336) with
    4-bit routed experts: the two chosen experts' dequantised weights, the
    oracle's gates and the dense SwiGLU give the reference."""
    w = WORKLOADS["mixtral_decode"]
    layer = make_checked_layer(w)
    a = OracleInputs(layer)
    dev = layer.to("cuda")
    cfg = B.config_of(w)
    q4 = B.quantize_experts_q4(dev)
    y = B.forward_q4(cfg, dev, q4)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    ids, gates, _, _ = oracle.route(ocfg(w), a.x, a.wr)
    X = dense.to_f64(a.x)
    y_ref = np.zeros((1, w.d))
    for j in range(w.k):
        e = int(ids[0, j])
        wg, wu, wd = (oracle.dequantize_q4(q4["q_" + n][e].cpu().numpy(), q4["s_" + n][e].cpu().numpy())
                      for n in ("gate", "up", "down"))
        y_ref += gates[0, j] * dense.dense_swiglu(X, wg, wu, wd)
    err = np.abs(y.float().cpu().numpy() - y_ref).max()
    assert err <= TOL * np.abs(y_ref).max(), err
