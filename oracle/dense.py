"""Numpy float64 restatements of the MoE layer, used only to pin the C oracle.

TEST INFRASTRUCTURE ONLY (see the package docstring).  Nothing here calls the
C oracle; both read the same stored bits and must agree to rounding.

* :func:`dense_forward` -- the dense formulation: every expert runs on every
  token and a [T, E] gate matrix that is zero outside each token's top-k masks
  the sum ("Small models, sparse experts", section "Dispatch decides
  everything": computing every expert and masking all but the top four;
  "Mixture-of-Experts -- more capacity per byte of weight", section "What's
  NOT shipped yet": every expert on every token, multiplied by the mostly-zero
  router weight).  Routing is written as matrix operations with a full
  lexicographic sort, not the C oracle's repeated selection.
* :func:`loop_over_experts_forward` -- the index_add formulation: for each
  expert that received tokens, gather its tokens, run the expert on them as one
  batch, scale by the gates and add into the output rows ("Small MoE
  Architecture, in depth", section "A small MoE layer in PyTorch").
* :func:`dense_swiglu` -- the textbook SwiGLU FFN down(silu(gate x) * up x)
  (the Expert module in the same section), for the E = 1, k = 1 special case.
"""
from __future__ import annotations

import numpy as np


def to_f64(a: np.ndarray) -> np.ndarray:
    """Stored bits -> float64: uint16 arrays are bf16 bit patterns, float32 as is."""
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if a.dtype == np.float32:
        return a.astype(np.float64)
    raise TypeError(a.dtype)


def _sigmoid(v):
    return 1.0 / (1.0 + np.exp(-v))


def _silu(u):
    return u * _sigmoid(u)


def score_matrix(X, Wr, score="softmax"):
    """The [T, E] score matrix: row-wise softmax of the logits X Wr^T, or their
    element-wise sigmoid."""
    L = X @ Wr.T
    if score == "sigmoid":
        return _sigmoid(L)
    Z = np.exp(L - L.max(axis=1, keepdims=True))
    return Z / Z.sum(axis=1, keepdims=True)


def route_matrix(X, Wr, k, score="softmax", norm_topk=True, bias=None):
    """Routing as matrix operations.  Returns (ids[T,k], gates[T,k], G[T,E]) where
    G is the dense gate matrix: G[t, ids[t,j]] = gates[t,j], zero elsewhere.
    With a balance bias [E] the selection key is the score plus the bias and the
    gates stay the unbiased scores ("Small MoE Architecture, in depth",
    SmallMoE.forward: topk of scores + balance_bias, gates gathered from scores)."""
    T, E = X.shape[0], Wr.shape[0]
    L = X @ Wr.T
    S = score_matrix(X, Wr, score)
    key = S if score == "sigmoid" else L
    if bias is not None:
        key = S + np.asarray(bias, np.float32).astype(np.float64)[None, :]
    # full sort by (key descending, expert index ascending)
    idx = np.broadcast_to(np.arange(E), (T, E))
    order = np.lexsort((idx, -key), axis=-1)
    ids = order[:, :k].astype(np.int32)
    gates = np.take_along_axis(S, ids, axis=1)
    if norm_topk:
        gates = gates / gates.sum(axis=1, keepdims=True)
    G = np.zeros((T, E))
    np.put_along_axis(G, ids.astype(np.int64), gates, axis=1)
    return ids, gates, G


def swiglu_act(X, Wg, Wu):
    """The expert's hidden activation silu(X Wg^T) * (X Wu^T) for X [n, d], Wg/Wu [h, d]."""
    return _silu(X @ Wg.T) * (X @ Wu.T)


def dense_swiglu(X, Wg, Wu, Wd):
    """down(silu(X Wg^T) * (X Wu^T)) for X [n, d], Wg/Wu [h, d], Wd [d, h]."""
    return swiglu_act(X, Wg, Wu) @ Wd.T


def dense_forward(cfg, x, wr, wg, wu, wd, shared=None, bias=None):
    """All experts on all tokens, masked by the gate matrix.  Returns (y[T,d], ids, gates)."""
    X, Wr = to_f64(x), to_f64(wr)
    ids, gates, G = route_matrix(X, Wr, cfg.k, cfg.score, cfg.norm_topk, bias)
    WG, WU, WD = to_f64(wg), to_f64(wu), to_f64(wd)
    Y = np.zeros((cfg.T, cfg.d))
    for e in range(cfg.E):
        Y += G[:, e:e + 1] * dense_swiglu(X, WG[e], WU[e], WD[e])
    if shared is not None and cfg.h_shared > 0:
        sg, su, sd, ws = (to_f64(a) for a in shared)
        Y += _sigmoid(X @ ws)[:, None] * dense_swiglu(X, sg, su, sd)
    return Y, ids, gates


def loop_over_experts_forward(cfg, x, wr, wg, wu, wd, shared=None, bias=None):
    """Per-expert gather / batch / index_add.  Returns y[T,d]."""
    X, Wr = to_f64(x), to_f64(wr)
    ids, gates, _ = route_matrix(X, Wr, cfg.k, cfg.score, cfg.norm_topk, bias)
    WG, WU, WD = to_f64(wg), to_f64(wu), to_f64(wd)
    out = np.zeros((cfg.T, cfg.d))
    if shared is not None and cfg.h_shared > 0:
        sg, su, sd, ws = (to_f64(a) for a in shared)
        out += _sigmoid(X @ ws)[:, None] * dense_swiglu(X, sg, su, sd)
    for e in np.unique(ids):
        tok, slot = np.nonzero(ids == e)
        ye = gates[tok, slot][:, None] * dense_swiglu(X[tok], WG[e], WU[e], WD[e])
        np.add.at(out, tok, ye)
    return out
