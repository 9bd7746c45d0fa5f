"""Parity of the CUDA path (through the C ABI) with the float64 oracle.

Routing outputs must match bit for bit (ids, counts, offsets, permutation),
gates and scores within 1e-6 absolute; layer outputs within
max|y - y_ref| <= 1e-2 * max|y_ref| (bf16 inputs, fp32 accumulation).  Inputs
are seeded and synthetic with the routing margin enforced (see support.py).
Full-size workloads are checked on every token for routing; the output is
checked on every token where the oracle affords it, and otherwise on tokens
chosen from the oracle's grouping so that every 64-row block of every
expert's segment (hence every 64-, 128- and 256-row GEMM tile, and the last
row of each segment) holds a checked row, plus seeded random tokens.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import dense
from sparse_mixture_experts_sigmoid_b200 import binding as B
from sparse_mixture_experts_sigmoid_b200 import synth
from sparse_mixture_experts_sigmoid_b200.workloads import WORKLOADS, Workload

from support import OracleInputs, enforce_margin, make_checked_layer, ocfg

pytestmark = pytest.mark.gpu

Y_TOL = 1e-2
GATE_TOL = 1e-6

_cache = {}


def checked(w: Workload):
    """(CPU layer with margins enforced, its device copy, oracle views), cached per workload."""
    key = w
    if key not in _cache:
        if len(_cache) > 2:       # keep host memory bounded across the full-size cases
            _cache.clear()
            torch.cuda.empty_cache()
        layer = make_checked_layer(w)
        _cache[key] = (layer, layer.to("cuda"), OracleInputs(layer))
    return _cache[key]


def tile_cover_tokens(w: Workload, ids_ref, block: int = 64, extra: int = 32):
    """Tokens whose assignments cover every `block`-row block of every expert's
    grouped segment (the first row of each segment and the last row of each
    block, so every segment's last row), plus `extra` seeded random tokens.
    Returns (tokens, {tile rows: fraction of tiles with a checked row})."""
    _, offsets, srt, _ = oracle.permute(ocfg(w), ids_ref)
    rows = []
    for e in range(w.E):
        b, en = int(offsets[e]), int(offsets[e + 1])
        if en > b:
            rows.append(b)
            rows.extend(min(s0 + block, en) - 1 for s0 in range(b, en, block))
    toks = set(int(srt[r]) // w.k for r in rows)
    rng = np.random.default_rng(4321)
    toks.update(int(t) for t in rng.choice(w.T, size=min(extra, w.T), replace=False))
    tokens = np.array(sorted(toks), dtype=np.int64)
    checked = np.zeros(w.T * w.k, bool)
    checked[np.isin(srt // w.k, tokens)] = True
    cover = {}
    for rb in (64, 128, 256):
        tiles = hit = 0
        for e in range(w.E):
            b, en = int(offsets[e]), int(offsets[e + 1])
            for s0 in range(b, en, rb):
                tiles += 1
                hit += bool(checked[s0:min(s0 + rb, en)].any())
        cover[rb] = hit / max(tiles, 1)
    return tokens, cover


def check_y(y_gpu: torch.Tensor, y_ref: np.ndarray, rows=None):
    y = y_gpu.float().cpu().numpy().astype(np.float64)
    if rows is not None:
        y = y[rows]
    scale = np.abs(y_ref).max()
    err = np.abs(y - y_ref).max()
    assert np.isfinite(y).all()
    assert scale > 0
    assert err <= Y_TOL * scale, f"max|y - y_ref| = {err:.3e} > {Y_TOL} * {scale:.3e}"
    return err / scale


def check_routing(w, a, ids, gates, sg=None, probs=None):
    c = ocfg(w)
    ids_ref, gates_ref, probs_ref, sg_ref = oracle.route(c, a.x, a.wr, a.w_sg, want_probs=probs is not None)
    np.testing.assert_array_equal(ids.cpu().numpy(), ids_ref)
    np.testing.assert_allclose(gates.cpu().numpy(), gates_ref, rtol=0, atol=GATE_TOL)
    if probs is not None:
        np.testing.assert_allclose(probs.cpu().numpy(), probs_ref, rtol=0, atol=GATE_TOL)
    if sg is not None:
        np.testing.assert_allclose(sg.cpu().numpy(), sg_ref, rtol=0, atol=GATE_TOL)
    return ids_ref


def check_permutation(w, ids_ref, counts, offsets, srt, inv):
    c_ref, o_ref, s_ref, i_ref = oracle.permute(ocfg(w), ids_ref)
    np.testing.assert_array_equal(counts.cpu().numpy(), c_ref)
    np.testing.assert_array_equal(offsets.cpu().numpy(), o_ref)
    np.testing.assert_array_equal(srt.cpu().numpy(), s_ref)
    np.testing.assert_array_equal(inv.cpu().numpy(), i_ref)


# ------------------------------------------------------------------ full-size workloads

FULL = ["tiny", "gemma_upcycle", "olmoe_zipf", "qwen_shared", "mixtral_prefill", "mixtral_decode"]
# outputs checked on every token; the other workloads use tile_cover_tokens
OUTPUT_ALL = {"tiny", "gemma_upcycle", "mixtral_decode"}


@pytest.mark.parametrize("name", FULL)
def test_full_size(name):
    w = WORKLOADS[name]
    layer, dev, a = checked(w)
    cfg = B.config_of(w)
    # stage entry points: router (with every score) and grouping, on all tokens
    ids, gates, probs, sg = B.route(cfg, dev.x, dev.w_router, dev.w_shared_gate, want_probs=True)
    torch.cuda.synchronize()
    ids_ref = check_routing(w, a, ids, gates, sg, probs)
    counts, offsets, srt, inv = B.permute(cfg, ids)
    torch.cuda.synchronize()
    check_permutation(w, ids_ref, counts, offsets, srt, inv)
    assert B.device_status() == 0
    del probs
    # the whole layer, in the launch configuration the benchmark times
    ws = B.alloc_workspace(cfg)
    y = B.forward_layer(cfg, dev, ws=ws)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    views = B.workspace_views(cfg, ws)
    check_routing(w, a, views["ids"], views["gates"], views["shared_gate"])
    check_permutation(w, ids_ref, views["counts"], views["offsets"], views["sorted_rows"], views["inv_rows"])
    if name in OUTPUT_ALL:
        rows = np.arange(w.T, dtype=np.int64)
    else:
        rows, cover = tile_cover_tokens(w, ids_ref)
        print(f"{name}: {rows.size} of {w.T} tokens checked; tiles with a checked row: "
              + ", ".join(f"{rb}-row {f:.3f}" for rb, f in cover.items()))
        assert all(f == 1.0 for f in cover.values()), cover
    y_ref = oracle.forward(ocfg(w), a.x, a.wr, a.wg, a.wu, a.wd, a.shared, tokens=rows)
    check_y(y, y_ref, rows)
    # a second call on the same workspace: same routing, output within tolerance
    ids_first = views["ids"].clone()
    y2 = B.forward_layer(cfg, dev, ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(ids_first, B.workspace_views(cfg, ws)["ids"])
    check_y(y2, y_ref, rows)


# ------------------------------------------------------------------ small shapes and edge cases

def small(name, **kw):
    base = dict(T=300, d=256, E=16, h=384, k=4, seed=50)
    base.update(kw)
    return Workload(name, **base)


SMALL = [
    small("ragged_softmax_norm"),
    small("ragged_softmax_nonorm", norm_topk=False, T=257, seed=51),
    small("sigmoid_norm", score="sigmoid", seed=52),
    small("sigmoid_nonorm", score="sigmoid", norm_topk=False, seed=53),
    small("shared_expert", h_shared=520, seed=54),
    small("f32_inputs", dtype="f32", seed=55),
    small("k1", k=1, seed=56),
    small("k_equals_E", E=6, k=6, seed=57),
    small("single_expert", E=1, k=1, seed=58),
    small("decode_T1", T=1, seed=59),
    small("decode_T3", T=3, E=64, k=8, seed=60),
    small("decode_T1_shared", T=1, h_shared=64, seed=65),
    small("decode_T1_ragged_widths", T=1, d=200, h=136, h_shared=72, score="sigmoid", seed=66),
    small("decode_T1_k16", T=1, E=64, k=16, d=128, h=64, router_std=0.2, seed=67),
    small("decode_T2_ragged_widths", T=2, d=200, h=136, seed=69),   # partial row block and reduction chunk
    small("decode_T16_k4", T=16, seed=70),   # 64 assignments: more work items than SMs in the batch-1 down kernel
    small("decode_T64_k1", T=64, k=1, d=512, h=1024, seed=71),   # the largest small batch, two 512-element chunks
    small("width_not_mult_64", d=200, h=136, seed=61),
    small("many_experts", E=512, k=16, T=200, d=128, h=64, router_std=0.2, seed=62),
    small("zipf_hot_expert", recipe="zipf", E=32, k=2, seed=63),
    small("f32_sigmoid_shared", dtype="f32", score="sigmoid", h_shared=64, seed=64),
    small("wide_model_width", d=832, h=256, seed=68),   # seven 128-column down tiles (column groups)
]


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_forward_small(w):
    layer, dev, a = checked(w)
    cfg = B.config_of(w)
    ws = B.alloc_workspace(cfg)
    y = B.forward_layer(cfg, dev, ws=ws)
    torch.cuda.synchronize()
    assert B.device_status() == 0
    views = B.workspace_views(cfg, ws)
    ids_ref = check_routing(w, a, views["ids"], views["gates"], views["shared_gate"])
    check_permutation(w, ids_ref, views["counts"], views["offsets"], views["sorted_rows"], views["inv_rows"])
    y_ref = oracle.forward(ocfg(w), a.x, a.wr, a.wg, a.wu, a.wd, a.shared)
    check_y(y, y_ref)


def test_one_expert_takes_every_token():
    """Router rows arranged so that expert 3 wins for every token: one segment
    holds all T rows and the other experts are empty (or nearly)."""
    w = small("all_to_one", T=520, E=8, k=1, seed=70)
    layer = synth.make_layer(w)
    layer.w_router[3] = layer.w_router[3] * 0 + 0.05
    layer.x[:, :] = layer.x.abs() + 0.1            # positive features: row 3 dominates
    enforce_margin(w, layer)
    a = OracleInputs(layer)
    dev = layer.to("cuda")
    cfg = B.config_of(w)
    ws = B.alloc_workspace(cfg)
    y = B.forward_layer(cfg, dev, ws=ws)
    torch.cuda.synchronize()
    views = B.workspace_views(cfg, ws)
    assert views["counts"][3].item() == w.T
    ids_ref = check_routing(w, a, views["ids"], views["gates"])
    check_permutation(w, ids_ref, views["counts"], views["offsets"], views["sorted_rows"], views["inv_rows"])
    check_y(y, oracle.forward(ocfg(w), a.x, a.wr, a.wg, a.wu, a.wd))


def test_stage_entry_points_compose_to_forward():
    """moe_route -> moe_permute -> moe_grouped_swiglu -> moe_combine equals moe_forward."""
    w = small("stages", T=333, seed=71)
    layer, dev, a = checked(w)
    cfg = B.config_of(w)
    ids, gates, _, _ = B.route(cfg, dev.x, dev.w_router)
    counts, offsets, srt, inv = B.permute(cfg, ids)
    act = B.grouped_swiglu(cfg, dev.x, dev.w_gate, dev.w_up, offsets, srt)
    y = B.combine(cfg, act, dev.w_down, offsets, srt, gates)
    y_fwd = B.forward_layer(cfg, dev)
    torch.cuda.synchronize()
    y_ref = oracle.forward(ocfg(w), a.x, a.wr, a.wg, a.wu, a.wd)
    check_y(y, y_ref)
    check_y(y_fwd, y_ref)
    # act rows are silu(W_gate[e] x_t) * (W_up[e] x_t) of the grouped rows, in
    # grouped order: every 5th grouped row and each segment's last row against
    # float64, within 1e-2 of the largest magnitude (act is stored in bf16)
    assert act.shape == (w.T * w.k, w.h)
    ids_ref, _, _, _ = oracle.route(ocfg(w), a.x, a.wr)
    _, off_ref, srt_ref, _ = oracle.permute(ocfg(w), ids_ref)
    np.testing.assert_array_equal(offsets.cpu().numpy(), off_ref)
    X, WG, WU = dense.to_f64(a.x), dense.to_f64(a.wg), dense.to_f64(a.wu)
    act_h = act.float().cpu().numpy().astype(np.float64)
    sel = sorted(set(range(0, w.T * w.k, 5)) | {int(o) - 1 for o in off_ref[1:] if o > 0})
    expert_of = np.searchsorted(off_ref, np.arange(w.T * w.k), side="right") - 1
    ref = np.stack([dense.swiglu_act(X[srt_ref[i] // w.k][None], WG[expert_of[i]], WU[expert_of[i]])[0]
                    for i in sel])
    got = act_h[sel]
    assert np.abs(got - ref).max() <= Y_TOL * np.abs(ref).max()


def test_permute_rejects_out_of_range_ids_on_device():
    """An expert id outside [0, E) is caught by the kernel's own range check:
    it reports MOE_ERR_DEVICE_INPUT and leaves every expert empty."""
    cfg = B.config(8, 64, 4, 64, 2)
    ids = torch.tensor([[0, 1]] * 7 + [[2, 9]], dtype=torch.int32, device="cuda")
    counts, offsets, srt, inv = B.permute(cfg, ids)
    assert B.device_status() == 6
    assert offsets.abs().sum().item() == 0 and counts.abs().sum().item() == 0
    assert B.device_status() == 0       # the flag was cleared


def test_zero_tokens():
    cfg = B.config(0, 64, 8, 128, 2)
    y = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")
    x = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")
    z = torch.zeros(8, 64, dtype=torch.bfloat16, device="cuda")
    wgt = torch.zeros(8, 128, 64, dtype=torch.bfloat16, device="cuda")
    wd = torch.zeros(8, 64, 128, dtype=torch.bfloat16, device="cuda")
    B.forward(cfg, x, z, wgt, wgt, wd, y=y, ws=torch.empty(256, dtype=torch.uint8, device="cuda"))
    torch.cuda.synchronize()
    assert B.device_status() == 0


def test_forward_with_nvtx_ranges_gives_the_same_bits():
    """moe_profile_nvtx only adds host-side ranges: y is bit-identical with them on."""
    w = SMALL[0]
    layer, dev, a = checked(w)
    cfg = B.config_of(w, combine="ordered")
    y0 = B.forward_layer(cfg, dev).cpu()
    B.profile_nvtx(True)
    try:
        y1 = B.forward_layer(cfg, dev).cpu()
    finally:
        B.profile_nvtx(False)
    assert B.device_status() == 0
    assert torch.equal(y0, y1)

