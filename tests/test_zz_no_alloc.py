"""moe_combine_noalloc, the combine entry point for callers that cannot
allocate device memory (its fp32 accumulator is a static device array inside
the library instead of a caller workspace).

Called through the C ABI and compared with moe_combine, the entry point that
takes a workspace, and with the float64 oracle's layer output, on two calls in
a row (the static array keeps the first call's sums, so the second call checks
that it is cleared).  This file is collected last so that a run stopping at the
first failure has already run every other test; it also passes on its own in a
fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from sparse_mixture_experts_sigmoid_b200 import binding as B
from sparse_mixture_experts_sigmoid_b200.workloads import Workload

from support import OracleInputs, make_checked_layer, ocfg

pytestmark = pytest.mark.gpu

Y_TOL = 1e-2   # the output tolerance of the parity tests: max|y - y_ref| <= 1e-2 * max|y_ref|

CASES = [
    Workload("noalloc_grouped", T=300, d=256, E=16, h=384, k=4, seed=80),                # tensor-core path
    Workload("noalloc_small", T=6, d=512, E=8, h=256, k=2, seed=81),                    # small-batch path
    Workload("noalloc_f32", T=100, d=128, E=8, h=128, k=2, dtype="f32", seed=82),
]


def _stages(w):
    cpu = make_checked_layer(w)      # routing margin enforced, so the oracle routes alike
    layer = cpu.to("cuda")
    cfg = B.config_of(w)
    ids, gates, _, _ = B.route(cfg, layer.x, layer.w_router)
    _, offsets, srt, _ = B.permute(cfg, ids)
    act = B.grouped_swiglu(cfg, layer.x, layer.w_gate, layer.w_up, offsets, srt)
    return cfg, cpu, layer, act, offsets, srt, gates


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_noalloc_matches_workspace_combine_twice(w):
    cfg, cpu, layer, act, offsets, srt, gates = _stages(w)
    y_ref = B.combine(cfg, act, layer.w_down, offsets, srt, gates).float()
    torch.cuda.synchronize()
    scale = y_ref.abs().max().item()
    assert scale > 0
    a = OracleInputs(cpu)
    y_oracle = oracle.forward(ocfg(w), a.x, a.wr, a.wg, a.wu, a.wd)
    o_scale = np.abs(y_oracle).max()
    for call in range(2):
        y = B.combine_noalloc(cfg, act, layer.w_down, offsets, srt, gates)
        torch.cuda.synchronize()
        assert B.device_status() == 0
        err = (y.float() - y_ref).abs().max().item()
        assert np.isfinite(err) and err <= Y_TOL * scale, f"call {call}: {err} > {Y_TOL} * {scale}"
        o_err = np.abs(y.float().cpu().numpy() - y_oracle).max()
        assert o_err <= Y_TOL * o_scale, f"call {call} vs oracle: {o_err} > {Y_TOL} * {o_scale}"


def test_noalloc_rejects_sizes_beyond_its_static_scratch():
    """T * d above the static accumulator's capacity is refused on the host."""
    limit = 4 << 20
    cfg = B.config(limit // 512 + 1, 512, 8, 64, 2)
    fake = ctypes.c_void_p(0x1000)
    st = B.lib().moe_combine_noalloc(ctypes.byref(cfg), fake, fake, fake, fake, fake, fake, None)
    assert st == 3    # MOE_ERR_WORKSPACE
