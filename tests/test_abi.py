"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/moe.h declares, and rejects bad arguments before
launching anything."""
import ctypes
import os
import re

import pytest

from sparse_mixture_experts_sigmoid_b200 import binding as B
from sparse_mixture_experts_sigmoid_b200.workloads import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include")) if f.endswith(".h")]


def declared_functions():
    names = set()
    for h in HEADERS:
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^\s*[A-Za-z_][\w\s\*]*?\b(moe_\w+)\s*\(", src, flags=re.M):
            names.add(m.group(1))
    return names


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert {"moe_route", "moe_permute", "moe_grouped_swiglu", "moe_combine", "moe_forward"} <= names
    L = B.lib()
    for n in sorted(names):
        assert hasattr(L, n), f"{n} declared in include/ but not exported"
    assert set(B.EXPORTED) <= names


def test_status_strings():
    for s in range(7):
        assert B.lib().moe_status_string(s).decode().startswith(B.STATUS_NAMES[s])
    assert b"unknown" in B.lib().moe_status_string(99)


@pytest.mark.parametrize("kw,status", [
    (dict(k=0), 1), (dict(k=9), 1), (dict(T=-1), 1), (dict(d=0), 1), (dict(score=2), 1),
    (dict(E=513, k=2), 2), (dict(k=17, E=32), 2), (dict(d=12), 2), (dict(h=100), 2),
    (dict(h_shared=12), 2), (dict(h_shared=-8), 1), (dict(T=1 << 30, k=4), 2), (dict(combine=2), 1),
    (dict(combine=-1), 1),
])
def test_validate_rejects(kw, status):
    base = dict(T=16, d=64, E=8, h=128, k=2, norm_topk=1, score=0, h_shared=0, dtype=0)
    base.update(kw)
    cfg = B.MoEConfig(**base)
    assert B.validate(cfg) == status


def test_validate_accepts_all_workloads():
    for w in WORKLOADS.values():
        assert B.validate(B.config_of(w)) == 0, w.name


def test_null_pointers_rejected_before_launch():
    cfg = B.config_of(WORKLOADS["tiny"])
    L = B.lib()
    P = ctypes.c_void_p
    fake = P(0x1000)
    assert L.moe_route(ctypes.byref(cfg), None, None, fake, None, fake, fake, None, None, None, 0, None) == 1
    assert L.moe_route(ctypes.byref(cfg), None, fake, fake, None, fake, fake, None, fake, None, 0, None) == 1  # no w_s
    big = B.config_of(WORKLOADS["olmoe_zipf"])
    # fp32 partial logits, one [T, 64] slab per chunk of the K range, then the
    # per-CTA score sums of the score-mean statistic ([T / 8, E] fp32)
    n = B.route_workspace_size(big)
    stats = 8192 // 8 * 64 * 4
    logits = n - stats
    assert logits >= 8192 * 64 * 4 and logits % (8192 * 64 * 4) == 0 and logits // (8192 * 64 * 4) <= 2048 // 64
    assert L.moe_route(ctypes.byref(big), None, fake, fake, None, fake, fake, None, None, None, 0, None) == 3
    assert L.moe_permute(ctypes.byref(cfg), fake, None, fake, fake, fake, fake, 1 << 20, None) == 1
    assert L.moe_permute(ctypes.byref(cfg), fake, fake, fake, fake, fake, None, 0, None) == 3
    assert L.moe_permute(ctypes.byref(cfg), fake, fake, fake, fake, fake, fake, 4, None) == 3
    assert L.moe_grouped_swiglu(ctypes.byref(cfg), fake, fake, None, fake, fake, fake, None) == 1
    assert L.moe_combine(ctypes.byref(cfg), fake, fake, fake, fake, fake, None, None, 0, None) == 1
    args = [fake] * 5 + [None] * 4 + [fake]
    assert L.moe_forward(ctypes.byref(cfg), None, *args, None, 0, None) == 3        # no workspace
    assert L.moe_forward(ctypes.byref(cfg), None, *args, P(0x10000), 16, None) == 3  # too small
    qcfg = B.config_of(WORKLOADS["qwen_shared"])
    assert L.moe_forward(ctypes.byref(qcfg), None, *args, P(0x10000), 1 << 40, None) == 1  # shared weights missing
    bf = B.config(16, 64, 8, 128, 2)
    assert L.moe_combine(ctypes.byref(bf), fake, fake, fake, fake, fake, fake, None, 0, None) == 3


def test_zero_tokens_is_a_no_op():
    cfg = B.config(0, 64, 8, 128, 2)
    P = ctypes.c_void_p
    assert B.lib().moe_route(ctypes.byref(cfg), None, None, None, None, None, None, None, None, None, 0, None) == 0
    assert B.lib().moe_forward(ctypes.byref(cfg), None, *([None] * 10), None, 0, None) == 0


def test_route_statistic_needs_its_workspace_part():
    """With a score-mean output the route scratch must also hold the per-CTA
    partial rows; without it the logits part alone suffices."""
    L = B.lib()
    fake = ctypes.c_void_p(0x1000)
    for T in (1, 64, 100, 4096):
        cfg = B.config(T, 256, 16, 128, 2)
        total = B.route_workspace_size(cfg)
        rows = T if T <= 64 else (T + 7) // 8
        assert total >= rows * 16 * 4
        opts = B.RouteOpts(None, 0x2000)
        ws = ctypes.c_void_p(1 << 20)
        assert L.moe_route(ctypes.byref(cfg), ctypes.byref(opts), fake, fake, None, fake, fake, None, None,
                           ws, total - 1, None) == 3
        assert L.moe_route(ctypes.byref(cfg), ctypes.byref(opts), fake, fake, None, fake, fake, None, None,
                           None, 0, None) == 3


def test_balance_entry_points_validate_on_the_host():
    L = B.lib()
    cfg = B.config(16, 64, 8, 128, 2)
    fake = ctypes.c_void_p(0x1000)
    assert L.moe_update_bias(ctypes.byref(cfg), None, ctypes.c_float(1e-3), fake, None) == 1
    assert L.moe_update_bias(ctypes.byref(cfg), fake, ctypes.c_float(float("nan")), fake, None) == 1
    assert L.moe_update_bias(ctypes.byref(cfg), fake, ctypes.c_float(float("inf")), fake, None) == 1
    assert L.moe_balance_loss(ctypes.byref(cfg), fake, fake, ctypes.c_float(0.01), None, None, None) == 1
    assert L.moe_balance_loss(ctypes.byref(cfg), fake, None, ctypes.c_float(0.01), None, fake, None) == 1
    bad = B.config(16, 64, 8, 128, 9)                      # k > E
    assert L.moe_update_bias(ctypes.byref(bad), fake, ctypes.c_float(1e-3), fake, None) == 1


def test_workspace_layout_is_disjoint_and_aligned():
    for w in WORKLOADS.values():
        cfg = B.config_of(w)
        n = B.workspace_size(cfg)
        base = 1 << 40
        v = B.WorkspaceViews()
        assert B.lib().moe_workspace_layout(ctypes.byref(cfg), ctypes.c_void_p(base), n, ctypes.byref(v)) == 0
        R = w.T * w.k
        esz = w.elem_bytes()
        sizes = {"ids": R * 4, "gates": R * 4, "shared_gate": w.T * 4 if w.h_shared else 0,
                 "counts": w.E * 4, "offsets": (w.E + 1) * 4, "sorted_rows": R * 4, "inv_rows": R * 4,
                 "act": R * w.h * esz, "act_shared": w.T * w.h_shared * esz,
                 "y_acc": w.T * w.d * 4 if w.dtype == "bf16" else 0}
        assert n >= sum(sizes.values()) + B.permute_workspace_size(cfg)
        spans = []
        for name, size in sizes.items():
            p = getattr(v, name)
            if size == 0:
                assert not p, name
                continue
            assert p % 256 == 0 and base <= p and p + size <= base + n, name
            spans.append((p, p + size))
        spans.sort()
        for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
            assert a1 <= b0
        # misaligned or short workspaces are refused
        assert B.lib().moe_workspace_layout(ctypes.byref(cfg), ctypes.c_void_p(base + 16), n,
                                            ctypes.byref(v)) == 3
        assert B.lib().moe_workspace_layout(ctypes.byref(cfg), ctypes.c_void_p(base), n - 1,
                                            ctypes.byref(v)) == 3


def test_workspace_never_holds_per_token_weight_copies():
    """The naive dispatch on "Small models, sparse experts" ("Dispatch decides
    everything") gathers each token's expert weights: a [2048, 512, 640] fp32
    tensor, 2.68 GB, for one projection of one layer.  The workspace here holds
    activations only and must stay orders of magnitude below that."""
    naive = 2048 * 512 * 640 * 4
    assert naive == 2_684_354_560
    w = WORKLOADS["gemma_upcycle"]
    assert B.workspace_size(B.config_of(w)) < naive / 50


def test_ordered_combine_workspace():
    """The ordered combine adds a [T*k, d] fp32 slot part to the workspace (and
    to the training workspace); moe_combine then needs T*k*d floats of ws."""
    L = B.lib()
    fake = ctypes.c_void_p(0x1000)
    for name in ("tiny", "olmoe_zipf", "mixtral_decode"):
        w = WORKLOADS[name]
        add, ordered = B.config_of(w), B.config_of(w, combine="ordered")
        slot = w.T * w.k * w.d * 4
        extra = B.workspace_size(ordered) - B.workspace_size(add)
        assert slot <= extra <= slot + 255
        if w.dtype == "bf16":
            extra_t = B.train_workspace_size(ordered) - B.train_workspace_size(add)
            assert slot <= extra_t <= slot + 255
        n = slot if w.dtype == "f32" else w.T * w.d * 4
        # the add mode's accumulator size is too small for the slot rows
        if w.k > 1:
            assert L.moe_combine(ctypes.byref(ordered), fake, fake, fake, fake, fake, fake, fake, w.T * w.d * 4,
                                 None) == 3
        assert L.moe_combine(ctypes.byref(ordered), fake, fake, fake, fake, fake, fake, None, 0, None) == 3
    with pytest.raises(ValueError):
        B.config(16, 64, 8, 128, 2, combine="sorted")



def test_profile_nvtx_is_host_only():
    """Turning the NVTX stage ranges on and off needs no GPU and never fails."""
    assert B.lib().moe_profile_nvtx(1) == 0
    assert B.lib().moe_profile_nvtx(0) == 0


def test_forward_host_workspace_and_argument_checks():
    """moe_forward_host's workspace holds the device copies of x and y plus the
    layer's workspace for one piece of ceil(T / chunks) tokens; chunks < 1 is
    rejected and chunks > T acts as T; bad arguments are caught on the host."""
    L = B.lib()
    fake = ctypes.c_void_p(0x1000)
    for name in ("tiny", "mixtral_prefill", "mixtral_decode"):
        w = WORKLOADS[name]
        cfg = B.config_of(w)
        esz = 4 if w.dtype == "f32" else 2
        rows = -(-w.T * w.d * esz // 256) * 256
        for chunks in (1, 2, 3, 4, 8):
            b = B.host_piece_bounds(w.T, chunks)
            assert b[0] == 0 and b[-1] == w.T and all(x <= y for x, y in zip(b, b[1:]))
            piece = max(y - x for x, y in zip(b, b[1:]))
            if len(b) > 3:   # three or more pieces: the outer ones hold about half the tokens
                assert abs(2 * (b[1] - b[0]) - (b[2] - b[1])) <= 2
            layer = B.workspace_size(B.config_of(w, T=piece))
            assert B.forward_host_workspace_size(cfg, chunks) == 2 * rows + layer
        assert B.forward_host_workspace_size(cfg, w.T + 5) == B.forward_host_workspace_size(cfg, min(w.T, 256))
        if w.T > 256:
            assert B.forward_host_workspace_size(cfg, 10**6) == B.forward_host_workspace_size(cfg, 256)
        n = ctypes.c_size_t(0)
        assert L.moe_forward_host_workspace_size(ctypes.byref(cfg), 0, ctypes.byref(n)) == 1
        assert L.moe_forward_host_workspace_size(ctypes.byref(cfg), -2, ctypes.byref(n)) == 1
        args = [fake] * 9
        # no x or y host buffer; no workspace; a misaligned workspace
        assert L.moe_forward_host(ctypes.byref(cfg), None, *args[1:], fake, 2, fake, 1 << 40, None, None) == 1
        assert L.moe_forward_host(ctypes.byref(cfg), *args, None, 2, fake, 1 << 40, None, None) == 1
        assert L.moe_forward_host(ctypes.byref(cfg), *args, fake, 2, None, 1 << 40, None, None) == 3
        assert L.moe_forward_host(ctypes.byref(cfg), *args, fake, 2, ctypes.c_void_p(0x1010), 1 << 40, None,
                                  None) == 3
        assert L.moe_forward_host(ctypes.byref(cfg), *args, fake, 2, fake, 16, None, None) == 3
        assert L.moe_forward_host(ctypes.byref(cfg), *args, fake, 0, fake, 1 << 40, None, None) == 1
