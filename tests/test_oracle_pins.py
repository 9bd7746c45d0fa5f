"""Pins of the float64 oracle to facts that do not come from the oracle itself.

* the routing worked example printed on "Tutorial 11: Mixture of Experts
  (MoE)", section 2 (golden file, run through the oracle's full route);
* the identity between "softmax over the kept scores" ("Small models, sparse
  experts", section "How it works") and full softmax + renormalisation;
* brute force over all k-subsets for the selected expert set;
* a full sort (numpy lexsort) for slot order and tie-breaking;
* the dense compute-all-experts-then-mask formulation and the
  loop-over-experts index_add formulation (numpy, float64, matrix ops);
* the E = 1, k = 1 special case, which is the textbook dense SwiGLU FFN;
* invariants: distinct ids, counts summing to T*k, a stable permutation
  (numpy's stable argsort), gates summing to one under renormalisation;
* selection with a balance bias and the bias update: hand-computed examples
  of "Small MoE Architecture, in depth" ("A small MoE layer in PyTorch"),
  brute force over k-subsets of the biased keys, and the dense and
  loop-over-experts formulations with the bias;
* the Switch statistics ("Mixture-of-Experts -- more capacity per byte of
  weight", "What's wired today"): a hand-computed example, the uniform router
  (P_e = 1/E) and uniform load (loss = alpha * k) closed forms, and the mean
  of the numpy score matrix;
* the backward pass: central finite differences of the oracle's own forward
  in float64 (every input element), and torch autograd (float64, CPU) on the
  dense all-experts-then-mask formulation.
"""
import itertools
import math
import os

import numpy as np
import pytest

import oracle
from oracle import dense
from sparse_mixture_experts_sigmoid_b200 import synth
from sparse_mixture_experts_sigmoid_b200.workloads import WORKLOADS, Workload

from support import OracleInputs, bits, ocfg

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

LIB_PATH = None  # the mutation tests rebind this to a mutated build


def lib():
    return oracle.load(LIB_PATH)


def _golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            out[key] = vals
    return out


# ---------------------------------------------------------------- worked example

def _worked_example_layer(norm):
    g = _golden("route_worked_example.txt")
    p = np.array([float(v) for v in g["probs"]])
    E, d = p.size, 8
    c = oracle.Cfg(T=1, d=d, E=E, h=8, k=int(g["top_k"][0]), norm_topk=norm, dtype="f32")
    x = np.zeros((1, d), np.float32)
    x[0, 0] = 1.0                                    # x = e_0, so logit_e = Wr[e, 0]
    wr = np.zeros((E, d), np.float32)
    wr[:, 0] = np.log(p).astype(np.float32)          # softmax(ln p) = p since sum(p) = 1
    return g, p, c, x, wr


def check_worked_example():
    g, p, c, x, wr = _worked_example_layer(norm=True)
    ids, gates, probs, _ = oracle.route(c, x, wr, want_probs=True, lib=lib())
    assert abs(p.sum() - 1.0) < 1e-15
    np.testing.assert_array_equal(ids[0], [int(v) for v in g["ids"]])
    num = [float(v) for v in g["normalised_exact_num"]]
    den = float(g["normalised_exact_den"][0])
    np.testing.assert_allclose(gates[0], np.array(num) / den, atol=1e-6)
    np.testing.assert_allclose(np.round(gates[0], 3), [float(v) for v in g["normalised"]], atol=0)
    np.testing.assert_allclose(probs[0], p, atol=1e-6)
    # the non-renormalised twin returns the raw probabilities of the kept experts
    _, _, c0, _, _ = _worked_example_layer(norm=False)
    ids0, gates0, _, _ = oracle.route(c0, x, wr, lib=lib())
    np.testing.assert_array_equal(ids0[0], ids[0])
    np.testing.assert_allclose(gates0[0], [float(v) for v in g["scores"]], atol=1e-6)


def test_worked_example():
    check_worked_example()


# ---------------------------------------------------------------- routing

def _random_case(rng, T, d, E, k, dtype="f32", score="softmax", norm=True, scale=1.0):
    c = oracle.Cfg(T=T, d=d, E=E, h=8, k=k, norm_topk=norm, score=score, dtype=dtype)
    x = (rng.standard_normal((T, d)) * scale).astype(np.float32)
    wr = (rng.standard_normal((E, d)) * 0.3).astype(np.float32)
    if dtype == "bf16":
        x = _to_bf16_bits(x)
        wr = _to_bf16_bits(wr)
    return c, x, wr


def _to_bf16_bits(a):
    u = np.ascontiguousarray(a, np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)   # round to nearest even
    return r


def check_routing_brute_force():
    rng = np.random.default_rng(11)
    for score in ("softmax", "sigmoid"):
        for E, k in [(5, 2), (6, 3), (4, 4), (7, 1)]:
            c, x, wr = _random_case(rng, 25, 9, E, k, score=score)
            ids, _, _, _ = oracle.route(c, x, wr, lib=lib())
            L = dense.to_f64(x) @ dense.to_f64(wr).T
            for t in range(c.T):
                # the kept set maximises the sum of logits over all k-subsets
                # (distinct continuous keys; sigmoid is monotone so the set is the same)
                best = max(itertools.combinations(range(E), k), key=lambda s: L[t, list(s)].sum())
                assert set(ids[t].tolist()) == set(best)
                # slots are ordered best first
                assert all(L[t, ids[t, j]] > L[t, ids[t, j + 1]] for j in range(k - 1))


def test_routing_brute_force():
    check_routing_brute_force()


def check_routing_vs_full_sort_and_ties():
    rng = np.random.default_rng(12)
    for score in ("softmax", "sigmoid"):
        for norm in (True, False):
            c, x, wr = _random_case(rng, 30, 16, 12, 4, score=score, norm=norm)
            # duplicate router rows -> exactly tied keys; ties go to the lower index
            wr[7] = wr[2]
            wr[9] = wr[2]
            wr[11] = wr[0]
            ids, gates, probs, _ = oracle.route(c, x, wr, want_probs=True, lib=lib())
            ids_ref, gates_ref, _ = dense.route_matrix(dense.to_f64(x), dense.to_f64(wr), c.k,
                                                       score, norm)
            np.testing.assert_array_equal(ids, ids_ref)
            np.testing.assert_allclose(gates, gates_ref, rtol=1e-13, atol=1e-15)
            for t in range(c.T):
                s = list(ids[t])
                for a, b in ((2, 7), (7, 9), (0, 11)):
                    if a in s and b in s:
                        assert s.index(a) < s.index(b)


def test_routing_vs_full_sort_and_ties():
    check_routing_vs_full_sort_and_ties()


def test_softmax_over_kept_equals_renormalised_softmax():
    """'softmax over those four scores' == full softmax then renormalise the kept."""
    rng = np.random.default_rng(13)
    c, x, wr = _random_case(rng, 64, 20, 16, 4, norm=True, scale=2.0)
    ids, gates, _, _ = oracle.route(c, x, wr, lib=lib())
    L = dense.to_f64(x) @ dense.to_f64(wr).T
    kept = np.take_along_axis(L, ids.astype(np.int64), axis=1)
    z = np.exp(kept - kept.max(axis=1, keepdims=True))
    np.testing.assert_allclose(gates, z / z.sum(axis=1, keepdims=True), rtol=0, atol=1e-15)
    np.testing.assert_allclose(gates.sum(axis=1), 1.0, atol=1e-15)


def check_margin():
    rng = np.random.default_rng(14)
    for score in ("softmax", "sigmoid"):
        c, x, wr = _random_case(rng, 20, 10, 9, 3, score=score)
        m = oracle.topk_margin(c, x, wr, lib=lib())
        L = dense.to_f64(x) @ dense.to_f64(wr).T
        key = 1.0 / (1.0 + np.exp(-L)) if score == "sigmoid" else L
        srt = -np.sort(-key, axis=1)[:, :c.k + 1]
        np.testing.assert_allclose(m, (srt[:, :-1] - srt[:, 1:]).min(axis=1), rtol=1e-12)


def test_margin():
    check_margin()


# ---------------------------------------------------------------- whole layer

SMALL_CASES = [
    # (T, d, E, h, k, score, norm, h_shared, dtype)
    (37, 24, 6, 20, 2, "softmax", True, 0, "f32"),
    (29, 16, 5, 12, 3, "softmax", False, 0, "bf16"),
    (31, 24, 7, 16, 2, "sigmoid", True, 0, "bf16"),
    (23, 16, 4, 20, 1, "sigmoid", False, 28, "f32"),
    (19, 32, 6, 8, 4, "softmax", False, 40, "bf16"),
]


def _small_layer(case, seed):
    T, d, E, h, k, score, norm, hs, dt = case
    w = Workload("small", T=T, d=d, E=E, h=h, k=k, score=score, norm_topk=norm, h_shared=hs,
                 dtype=dt, seed=seed, router_std=0.3, weight_std=0.3)
    return w, OracleInputs(synth.make_layer(w, "cpu"))


def check_dense_formulation():
    for i, case in enumerate(SMALL_CASES):
        w, a = _small_layer(case, 100 + i)
        c = ocfg(w)
        y = oracle.forward(c, a.x, a.wr, a.wg, a.wu, a.wd, a.shared, lib=lib())
        y_ref, ids_ref, gates_ref = dense.dense_forward(c, a.x, a.wr, a.wg, a.wu, a.wd, a.shared)
        scale = np.abs(y_ref).max()
        assert scale > 0
        np.testing.assert_allclose(y, y_ref, rtol=0, atol=1e-12 * scale)
        ids, gates, _, sg = oracle.route(c, a.x, a.wr, a.w_sg, lib=lib())
        np.testing.assert_array_equal(ids, ids_ref)
        np.testing.assert_allclose(gates, gates_ref, rtol=1e-13, atol=1e-15)
        if w.h_shared:
            sg_ref = 1.0 / (1.0 + np.exp(-(dense.to_f64(a.x) @ dense.to_f64(a.w_sg))))
            np.testing.assert_allclose(sg, sg_ref, rtol=1e-13)


def test_dense_formulation():
    check_dense_formulation()


def check_tiny_workload():
    w = WORKLOADS["tiny"]
    a = OracleInputs(synth.make_layer(w, "cpu"))
    c = ocfg(w)
    y = oracle.forward(c, a.x, a.wr, a.wg, a.wu, a.wd, lib=lib())
    y_dense, _, _ = dense.dense_forward(c, a.x, a.wr, a.wg, a.wu, a.wd)
    y_loop = dense.loop_over_experts_forward(c, a.x, a.wr, a.wg, a.wu, a.wd)
    scale = np.abs(y_dense).max()
    np.testing.assert_allclose(y, y_dense, rtol=0, atol=1e-12 * scale)
    np.testing.assert_allclose(y, y_loop, rtol=0, atol=1e-12 * scale)
    # a subset of tokens evaluates to the same rows
    sub = np.array([63, 0, 17], np.int64)
    np.testing.assert_allclose(oracle.forward(c, a.x, a.wr, a.wg, a.wu, a.wd, tokens=sub,
                                              lib=lib()), y[sub], rtol=0, atol=0)


def test_tiny_workload_three_formulations():
    check_tiny_workload()


def check_loop_over_experts():
    for i, case in enumerate(SMALL_CASES[:3] + SMALL_CASES[4:]):
        w, a = _small_layer(case, 200 + i)
        c = ocfg(w)
        y = oracle.forward(c, a.x, a.wr, a.wg, a.wu, a.wd, a.shared, lib=lib())
        y_ref = dense.loop_over_experts_forward(c, a.x, a.wr, a.wg, a.wu, a.wd, a.shared)
        np.testing.assert_allclose(y, y_ref, rtol=0, atol=1e-12 * np.abs(y_ref).max())


def test_loop_over_experts():
    check_loop_over_experts()


def check_single_expert_is_dense_swiglu():
    for score, norm in (("softmax", False), ("softmax", True), ("sigmoid", True)):
        w = Workload("one", T=17, d=24, E=1, h=40, k=1, score=score, norm_topk=norm,
                     dtype="f32", seed=7, weight_std=0.3, router_std=0.3)
        a = OracleInputs(synth.make_layer(w, "cpu"))
        c = ocfg(w)
        y = oracle.forward(c, a.x, a.wr, a.wg, a.wu, a.wd, lib=lib())
        ref = dense.dense_swiglu(dense.to_f64(a.x), dense.to_f64(a.wg[0]), dense.to_f64(a.wu[0]),
                                 dense.to_f64(a.wd[0]))
        np.testing.assert_allclose(y, ref, rtol=0, atol=1e-12 * np.abs(ref).max())
        ids, gates, _, _ = oracle.route(c, a.x, a.wr, lib=lib())
        assert (ids == 0).all() and np.all(gates == 1.0)
    # sigmoid without renormalisation: gate = sigmoid(logit)
    w = Workload("one", T=9, d=16, E=1, h=8, k=1, score="sigmoid", norm_topk=False, dtype="f32",
                 seed=8, weight_std=0.3, router_std=0.3)
    a = OracleInputs(synth.make_layer(w, "cpu"))
    c = ocfg(w)
    y = oracle.forward(c, a.x, a.wr, a.wg, a.wu, a.wd, lib=lib())
    l = dense.to_f64(a.x) @ dense.to_f64(a.wr[0])
    ref = (1 / (1 + np.exp(-l)))[:, None] * dense.dense_swiglu(
        dense.to_f64(a.x), dense.to_f64(a.wg[0]), dense.to_f64(a.wu[0]), dense.to_f64(a.wd[0]))
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-12 * np.abs(ref).max())


def test_single_expert_is_dense_swiglu():
    check_single_expert_is_dense_swiglu()


# ---------------------------------------------------------------- grouping invariants

def check_permutation_invariants():
    rng = np.random.default_rng(15)
    for T, E, k in [(50, 7, 3), (1, 4, 4), (64, 8, 2), (40, 16, 1)]:
        c = oracle.Cfg(T=T, d=8, E=E, h=8, k=k)
        # distinct ids per token, skewed towards expert 0 so some experts are empty
        ids = np.stack([rng.choice(E, size=k, replace=False,
                                   p=np.r_[0.5, np.full(E - 1, 0.5 / (E - 1))])
                        for _ in range(T)]).astype(np.int32)
        counts, offsets, srt, inv = oracle.permute(c, ids, lib=lib())
        flat = ids.reshape(-1)
        np.testing.assert_array_equal(counts, np.bincount(flat, minlength=E))
        assert counts.sum() == T * k
        np.testing.assert_array_equal(offsets, np.r_[0, np.cumsum(counts)])
        np.testing.assert_array_equal(srt, np.argsort(flat, kind="stable"))
        np.testing.assert_array_equal(inv[srt], np.arange(T * k))
        for e in range(E):
            seg = srt[offsets[e]:offsets[e + 1]]
            assert (flat[seg] == e).all()


def test_permutation_invariants():
    check_permutation_invariants()


def test_route_invariants_on_workload_shapes():
    """Distinct ids, renormalised gates sum to one, unnormalised sum below one."""
    for name in ("tiny", "gemma_upcycle"):
        w = WORKLOADS[name].with_(T=48)
        layer = synth.make_layer(w, "cpu")
        c = ocfg(w)
        ids, gates, _, _ = oracle.route(c, bits(layer.x), bits(layer.w_router))
        for t in range(w.T):
            assert len(set(ids[t].tolist())) == w.k
        s = gates.sum(axis=1)
        if w.norm_topk:
            np.testing.assert_allclose(s, 1.0, atol=1e-12)
        else:
            assert (s < 1.0).all()


def test_oracle_rejects_bad_arguments():
    c = oracle.Cfg(T=2, d=4, E=3, h=4, k=4, dtype="f32")        # k > E
    x = np.zeros((2, 4), np.float32)
    wr = np.zeros((3, 4), np.float32)
    with pytest.raises(ValueError):
        oracle.route(c, x, wr)
    c = oracle.Cfg(T=1, d=4, E=3, h=4, k=1)
    with pytest.raises(ValueError):
        oracle.permute(c, np.array([3], np.int32))                 # id out of range


# ---------------------------------------------------------------- balance bias and Switch statistics

def _bias_example(norm=True, bias=True):
    g = _golden("balance_bias_example.txt")
    s = np.array([float(v) for v in g["scores"]])
    E, d = s.size, 4
    c = oracle.Cfg(T=1, d=d, E=E, h=8, k=int(g["top_k"][0]), norm_topk=norm, score="sigmoid", dtype="f32")
    x = np.zeros((1, d), np.float32)
    x[0, 0] = 1.0                                              # logit_e = Wr[e, 0]
    wr = np.zeros((E, d), np.float32)
    wr[:, 0] = np.log(s / (1.0 - s)).astype(np.float32)       # sigmoid(logit(s)) = s
    b = np.array([float(v) for v in g["bias"]], np.float32) if bias else None
    return g, c, x, wr, b


def check_balance_bias_example():
    g, c, x, wr, b = _bias_example()
    ids, gates, probs, _ = oracle.route(c, x, wr, want_probs=True, bias=b, lib=lib())
    np.testing.assert_array_equal(ids[0], [int(v) for v in g["ids"]])
    np.testing.assert_allclose(gates[0], [float(v) for v in g["gates_normalised"]], atol=1e-6)
    np.testing.assert_allclose(probs[0], [float(v) for v in g["scores"]], atol=1e-6)   # scores stay unbiased
    _, c0, _, _, _ = _bias_example(norm=False)
    ids0, gates0, _, _ = oracle.route(c0, x, wr, bias=b, lib=lib())
    np.testing.assert_array_equal(ids0[0], ids[0])
    np.testing.assert_allclose(gates0[0], [float(v) for v in g["gates_raw"]], atol=1e-6)
    idsu, gatesu, _, _ = oracle.route(c, x, wr, lib=lib())
    np.testing.assert_array_equal(idsu[0], [int(v) for v in g["ids_unbiased"]])
    np.testing.assert_allclose(gatesu[0], [float(v) for v in g["gates_unbiased_normalised"]], atol=1e-6)
    # the margin sees the biased keys: 0.95 - 0.9 and 0.9 - 0.8 -> 0.05
    m = oracle.topk_margin(c, x, wr, bias=b, lib=lib())
    np.testing.assert_allclose(m, [0.05], atol=1e-6)


def test_balance_bias_example():
    check_balance_bias_example()


def check_biased_routing_brute_force_and_formulations():
    rng = np.random.default_rng(21)
    for score in ("sigmoid", "softmax"):
        for norm in (True, False):
            c, x, wr = _random_case(rng, 30, 12, 9, 3, score=score, norm=norm)
            # biases of the size of the score spread, so they change many choices
            b = (rng.standard_normal(9) * (0.3 if score == "sigmoid" else 0.1)).astype(np.float32)
            ids, gates, _, _ = oracle.route(c, x, wr, bias=b, lib=lib())
            ids_plain, _, _, _ = oracle.route(c, x, wr, lib=lib())
            assert (ids != ids_plain).any(), "the bias should change some selections"
            S = dense.score_matrix(dense.to_f64(x), dense.to_f64(wr), score)
            key = S + b.astype(np.float64)[None, :]
            for t in range(c.T):
                best = max(itertools.combinations(range(c.E), c.k), key=lambda s_: key[t, list(s_)].sum())
                assert set(ids[t].tolist()) == set(best)
                assert all(key[t, ids[t, j]] > key[t, ids[t, j + 1]] for j in range(c.k - 1))
                g = S[t, ids[t]]
                np.testing.assert_allclose(gates[t], g / g.sum() if norm else g, rtol=1e-13, atol=1e-15)
    # the whole layer with a bias: C loop == dense masking == loop over experts
    w, a = _small_layer((27, 16, 7, 12, 2, "sigmoid", True, 12, "bf16"), 300)
    c = ocfg(w)
    b = (np.random.default_rng(22).standard_normal(w.E) * 0.3).astype(np.float32)
    y = oracle.forward(c, a.x, a.wr, a.wg, a.wu, a.wd, a.shared, bias=b, lib=lib())
    y_dense, ids_d, _ = dense.dense_forward(c, a.x, a.wr, a.wg, a.wu, a.wd, a.shared, bias=b)
    y_loop = dense.loop_over_experts_forward(c, a.x, a.wr, a.wg, a.wu, a.wd, a.shared, bias=b)
    scale = np.abs(y_dense).max()
    np.testing.assert_allclose(y, y_dense, rtol=0, atol=1e-12 * scale)
    np.testing.assert_allclose(y, y_loop, rtol=0, atol=1e-12 * scale)
    ids, _, _, _ = oracle.route(c, a.x, a.wr, a.w_sg, bias=b, lib=lib())
    np.testing.assert_array_equal(ids, ids_d)


def test_biased_routing_brute_force_and_formulations():
    check_biased_routing_brute_force_and_formulations()


def check_bias_update_example():
    g = _golden("bias_update_example.txt")
    E, T, k = int(g["E"][0]), int(g["T"][0]), int(g["top_k"][0])
    c = oracle.Cfg(T=T, d=8, E=E, h=8, k=k)
    counts = np.array([int(v) for v in g["counts"]], np.int32)
    assert counts.sum() == T * k
    before = np.array([float(v) for v in g["bias_before"]], np.float32)
    after = oracle.update_bias(c, counts, float(g["lr"][0]), before, lib=lib())
    np.testing.assert_array_equal(after, np.array([float(v) for v in g["bias_after"]], np.float32))
    # an exactly balanced load leaves the bias unchanged; a second step moves it again
    np.testing.assert_array_equal(oracle.update_bias(c, np.full(E, 3, np.int32), 0.001, before, lib=lib()),
                                  before)
    twice = oracle.update_bias(c, counts, 0.001, after, lib=lib())
    np.testing.assert_allclose(twice - before, [-0.002, 0.002, 0.0, 0.0], atol=1e-9)


def test_bias_update_example():
    check_bias_update_example()


def check_switch_statistics():
    g = _golden("switch_balance_example.txt")
    E, T, k = int(g["E"][0]), int(g["T"][0]), int(g["top_k"][0])
    c = oracle.Cfg(T=T, d=T, E=E, h=8, k=k, norm_topk=False, dtype="f32")
    x = np.eye(T, dtype=np.float32)                            # token t reads router column t
    wr = np.zeros((E, T), np.float32)
    for t in range(T):
        wr[:, t] = np.log([float(v) for v in g[f"probs_t{t}"]]).astype(np.float32)
    ids, _, _, _ = oracle.route(c, x, wr, lib=lib())
    counts, _, _, _ = oracle.permute(c, ids, lib=lib())
    np.testing.assert_array_equal(counts, [int(v) for v in g["counts"]])
    P = oracle.score_mean(c, x, wr, lib=lib())
    np.testing.assert_allclose(P, [float(v) for v in g["P"]], atol=1e-7)
    loss, f = oracle.balance_loss(c, counts, P, float(g["alpha"][0]), lib=lib())
    np.testing.assert_allclose(f, [float(v) for v in g["f"]], rtol=0, atol=0)
    np.testing.assert_allclose(loss, float(g["loss"][0]), rtol=1e-6)
    # closed forms: a zero router gives every expert the score 1/E (softmax) or
    # 1/2 (sigmoid); a uniform load then gives alpha * k
    for score, p in (("softmax", 1 / 8), ("sigmoid", 0.5)):
        c8 = oracle.Cfg(T=16, d=4, E=8, h=8, k=2, score=score, dtype="f32")
        xz = np.random.default_rng(3).standard_normal((16, 4)).astype(np.float32)
        P8 = oracle.score_mean(c8, xz, np.zeros((8, 4), np.float32), lib=lib())
        np.testing.assert_allclose(P8, np.full(8, p), rtol=1e-15)
    c8 = oracle.Cfg(T=16, d=4, E=8, h=8, k=2, dtype="f32")
    loss8, f8 = oracle.balance_loss(c8, np.full(8, 4, np.int32), np.full(8, 1 / 8), 0.01, lib=lib())
    np.testing.assert_allclose(f8, np.full(8, 0.25), rtol=0)
    np.testing.assert_allclose(loss8, 0.01 * 2, rtol=1e-15)
    # random router: the mean of the score matrix
    rng = np.random.default_rng(23)
    for score in ("softmax", "sigmoid"):
        cr, xr, wrr = _random_case(rng, 40, 10, 6, 2, score=score, dtype="bf16")
        Pr = oracle.score_mean(cr, xr, wrr, lib=lib())
        S = dense.score_matrix(dense.to_f64(xr), dense.to_f64(wrr), score)
        np.testing.assert_allclose(Pr, S.mean(axis=0), rtol=1e-13)


def test_switch_statistics():
    check_switch_statistics()


# ---------------------------------------------------------------- backward

BWD_CASES = [
    # (T, d, E, h, k, score, norm, h_shared, biased)
    (5, 6, 4, 5, 2, "softmax", True, 0, False),
    (4, 5, 5, 4, 3, "softmax", False, 3, False),
    (5, 6, 4, 5, 2, "sigmoid", True, 3, True),
    (4, 6, 3, 4, 1, "sigmoid", False, 0, False),
    (3, 4, 1, 3, 1, "softmax", True, 2, False),      # E = 1: the gate is constant 1
]


def _bwd_case(case, seed):
    """float64 inputs of a small layer with every token's selection margin >= 1e-3."""
    T, d, E, h, k, score, norm, hs, biased = case
    rng = np.random.default_rng(seed)
    c = oracle.Cfg(T=T, d=d, E=E, h=h, k=k, norm_topk=norm, score=score, h_shared=hs, dtype="f64")
    wr = rng.standard_normal((E, d)) * 0.7
    b = (rng.standard_normal(E) * 0.1).astype(np.float32) if biased else None
    x = rng.standard_normal((T, d))
    for _ in range(200):
        m = oracle.topk_margin(c, x, wr, bias=b, lib=lib())
        bad = ~(m >= 1e-3)
        if not bad.any():
            break
        x[bad] = rng.standard_normal((int(bad.sum()), d))
    t = {"x": x, "wr": wr, "wg": rng.standard_normal((E, h, d)) * 0.5, "wu": rng.standard_normal((E, h, d)) * 0.5,
         "wd": rng.standard_normal((E, d, h)) * 0.5, "dy": rng.standard_normal((T, d))}
    if hs:
        t.update(shg=rng.standard_normal((hs, d)) * 0.5, shu=rng.standard_normal((hs, d)) * 0.5,
                 shd=rng.standard_normal((d, hs)) * 0.5, ws=rng.standard_normal(d) * 0.5)
    return c, t, b


def _fwd_loss(c, t, b):
    sh = (t["shg"], t["shu"], t["shd"], t["ws"]) if c.h_shared else None
    y = oracle.forward(c, t["x"], t["wr"], t["wg"], t["wu"], t["wd"], sh, bias=b, nthreads=1, lib=lib())
    return float((y * t["dy"]).sum())


_GRAD_OF = {"x": "dx", "wr": "dw_router", "wg": "dw_gate", "wu": "dw_up", "wd": "dw_down",
            "shg": "dsh_gate", "shu": "dsh_up", "shd": "dsh_down", "ws": "dw_shared_gate"}


def _oracle_grads(c, t, b):
    sh = (t["shg"], t["shu"], t["shd"], t["ws"]) if c.h_shared else None
    return oracle.backward(c, t["x"], t["wr"], t["wg"], t["wu"], t["wd"], t["dy"], sh, bias=b, lib=lib())


def check_backward_finite_differences():
    for i, case in enumerate(BWD_CASES):
        c, t, b = _bwd_case(case, 500 + i)
        g = _oracle_grads(c, t, b)
        for name, gname in _GRAD_OF.items():
            if name not in t:
                continue
            arr = t[name]
            fd = np.zeros_like(arr)
            for idx in np.ndindex(arr.shape):
                v = arr[idx]
                eps = 1e-6 * max(1.0, abs(v))
                arr[idx] = v + eps
                lp = _fwd_loss(c, t, b)
                arr[idx] = v - eps
                lm = _fwd_loss(c, t, b)
                arr[idx] = v
                fd[idx] = (lp - lm) / (2 * eps)
            scale = max(np.abs(fd).max(), 1e-3)
            np.testing.assert_allclose(g[gname], fd, rtol=0, atol=1e-6 * scale, err_msg=f"case {i} {gname}")


def test_backward_finite_differences():
    check_backward_finite_differences()


def _torch_dense_grads(c, t, b):
    """Autograd of the dense all-experts-then-mask formulation (float64, CPU)."""
    import torch
    T_ = {k_: torch.tensor(v, dtype=torch.float64, requires_grad=(k_ != "dy")) for k_, v in t.items()}
    X, Wr = T_["x"], T_["wr"]
    L = X @ Wr.T
    S = torch.sigmoid(L) if c.score == "sigmoid" else torch.softmax(L, dim=1)
    key = (S if c.score == "sigmoid" else L).detach().numpy()
    if b is not None:
        key = S.detach().numpy() + b.astype(np.float64)[None, :]
    idx = np.broadcast_to(np.arange(c.E), key.shape)
    order = torch.tensor(np.lexsort((idx, -key), axis=-1)[:, :c.k].copy())
    gates = S.gather(1, order)
    if c.norm_topk:
        gates = gates / gates.sum(dim=1, keepdim=True)
    G = torch.zeros(c.T, c.E, dtype=torch.float64).scatter(1, order, gates)
    Y = torch.zeros(c.T, c.d, dtype=torch.float64)
    for e in range(c.E):
        a = torch.nn.functional.silu(X @ T_["wg"][e].T) * (X @ T_["wu"][e].T)
        Y = Y + G[:, e:e + 1] * (a @ T_["wd"][e].T)
    if c.h_shared:
        a = torch.nn.functional.silu(X @ T_["shg"].T) * (X @ T_["shu"].T)
        Y = Y + torch.sigmoid(X @ T_["ws"])[:, None] * (a @ T_["shd"].T)
    (Y * T_["dy"]).sum().backward()
    return {_GRAD_OF[k_]: v.grad.numpy() for k_, v in T_.items() if k_ != "dy"}


def check_backward_vs_autograd_dense():
    for i, case in enumerate(BWD_CASES):
        c, t, b = _bwd_case(case, 600 + i)
        g = _oracle_grads(c, t, b)
        ref = _torch_dense_grads(c, t, b)
        for gname, r in ref.items():
            scale = max(np.abs(r).max(), 1e-12)
            np.testing.assert_allclose(g[gname], r, rtol=0, atol=1e-12 * scale, err_msg=f"case {i} {gname}")


def test_backward_vs_autograd_dense():
    check_backward_vs_autograd_dense()


# ---------------------------------------------------------------- 4-bit routed experts

def check_q4_group_example():
    g = _golden("q4_group_example.txt")
    w = np.zeros((1, 64), np.float32)
    w[0, :8] = [float(v) for v in g["weights"]]
    for stored in (w, _to_bf16_bits(w)):
        q, sc = oracle.quantize_q4(stored, lib=lib())
        assert sc.shape == (1, 1) and sc[0, 0] == float(g["scale"][0])
        np.testing.assert_array_equal(q[0, :4], [int(b, 16) for b in g["bytes"]])
        assert (q[0, 4:] == 0x88).all()          # zeros: code 0, nibble 8
        deq = oracle.dequantize_q4(q, sc, lib=lib())
        np.testing.assert_array_equal(deq[0, :8], [float(v) for v in g["dequantised"]])
        assert (deq[0, 8:] == 0).all()
    # a group of zeros: scale 0, codes 0
    q, sc = oracle.quantize_q4(np.zeros((2, 128), np.float32), lib=lib())
    assert (sc == 0).all() and (q == 0x88).all()


def test_q4_group_example():
    check_q4_group_example()


def check_q4_nearest_code():
    """Every code is the nearest of -7..7 to w / scale in fp32 (ties to the even
    code), the scale is fp32(max|w|) / 7 in fp32, and every represented value is
    within half a scale of the weight."""
    rng = np.random.default_rng(31)
    w = (rng.standard_normal((6, 192)) * rng.uniform(0.01, 3.0, (6, 1))).astype(np.float32)
    w[2, 64:128] *= 0                           # one all-zero group
    q, sc = oracle.quantize_q4(w, lib=lib())
    deq = oracle.dequantize_q4(q, sc, lib=lib())
    cand = np.arange(-7, 8, dtype=np.float64)
    for r in range(w.shape[0]):
        for gi in range(3):
            grp = w[r, 64 * gi:64 * gi + 64]
            s_ref = np.float32(np.abs(grp).max()) / np.float32(7)
            assert sc[r, gi] == s_ref
            nib = np.stack([q[r, 32 * gi:32 * gi + 32] & 15, q[r, 32 * gi:32 * gi + 32] >> 4], 1).reshape(-1)
            codes = nib.astype(np.int64) - 8
            for i, v in enumerate(grp):
                if s_ref == 0:
                    assert codes[i] == 0
                    continue
                ratio = np.float64(np.float32(v) / s_ref)
                dist = np.abs(cand - ratio)
                best = cand[dist == dist.min()]
                want = best[0] if best.size == 1 else best[np.abs(best) % 2 == 0][0]
                assert codes[i] == want, (r, gi, i)
            assert np.all(np.abs(deq[r, 64 * gi:64 * gi + 64] - grp) <= s_ref / 2 * (1 + 1e-6))


def test_q4_nearest_code():
    check_q4_nearest_code()


def check_q4_forward_is_the_dense_layer_on_the_represented_weights():
    from oracle import dense
    w, a = _small_layer((21, 64, 5, 128, 2, "softmax", True, 64, "bf16"), 700)
    c = ocfg(w)
    qs = [oracle.quantize_q4(t, lib=lib()) for t in (a.wg, a.wu, a.wd)]
    y = oracle.forward_q4(c, a.x, a.wr, *qs[0], *qs[1], *qs[2], a.shared, lib=lib())
    deq = [oracle.dequantize_q4(q, s_, lib=lib()) for q, s_ in qs]
    X, Wr = dense.to_f64(a.x), dense.to_f64(a.wr)
    _, _, G = dense.route_matrix(X, Wr, c.k, c.score, c.norm_topk)
    Y = np.zeros((c.T, c.d))
    for e in range(c.E):
        Y += G[:, e:e + 1] * dense.dense_swiglu(X, deq[0][e], deq[1][e], deq[2][e])
    sg, su, sd, ws = (dense.to_f64(t) for t in a.shared)
    Y += 1 / (1 + np.exp(-(X @ ws)))[:, None] * dense.dense_swiglu(X, sg, su, sd)
    np.testing.assert_allclose(y, Y, rtol=0, atol=1e-12 * np.abs(Y).max())


def test_q4_forward_is_the_dense_layer_on_the_represented_weights():
    check_q4_forward_is_the_dense_layer_on_the_represented_weights()


# The checks the mutation tests run against deliberately broken builds.
PIN_CHECKS = [check_worked_example, check_routing_brute_force, check_routing_vs_full_sort_and_ties,
              check_margin, check_dense_formulation, check_tiny_workload, check_loop_over_experts,
              check_single_expert_is_dense_swiglu, check_permutation_invariants, check_balance_bias_example,
              check_biased_routing_brute_force_and_formulations, check_bias_update_example,
              check_switch_statistics, check_backward_finite_differences, check_backward_vs_autograd_dense,
              check_q4_group_example, check_q4_nearest_code,
              check_q4_forward_is_the_dense_layer_on_the_represented_weights]

assert math.isclose(64 ** (1 / 3), 4.0)
