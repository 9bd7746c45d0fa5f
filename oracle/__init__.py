"""Float64 CPU oracle for the top-k routed MoE SwiGLU FFN forward pass.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
timed CPU baseline may import this package.  The product path (the CUDA
library and its Python binding) never imports it, and it imports nothing from
the product: the two meet only at the seeded input generator, whose tensors
both consume.

Two independent formulations live here:

* ``moe_oracle.c`` -- a plain per-token float64 loop in C (OpenMP over tokens):
  routing, grouping and the expert SwiGLU/combine.  This is THE oracle.
* ``dense.py`` -- numpy float64 restatements used only to pin the C oracle:
  the dense compute-all-experts-then-mask formulation ("Small models, sparse
  experts", section "Dispatch decides everything"; "Mixture-of-Experts -- more
  capacity per byte of weight", section "What's NOT shipped yet"), and the
  loop-over-experts index_add formulation ("Small MoE Architecture, in depth",
  section "A small MoE layer in PyTorch").

Inputs are numpy arrays holding the stored bits: ``uint16`` for bf16 tensors,
``float32`` for fp32 tensors, C-contiguous.  All results are float64 (ids and
permutations int32).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

SOFTMAX, SIGMOID = 0, 1
BF16, F32, F64 = 0, 1, 2


@dataclass(frozen=True)
class Cfg:
    """Layer shape and options as the oracle sees them."""
    T: int
    d: int
    E: int
    h: int
    k: int
    norm_topk: bool = True
    score: str = "softmax"      # "softmax" | "sigmoid"
    h_shared: int = 0
    dtype: str = "bf16"         # "bf16" | "f32" | "f64" (f64: pins only)


class _CCfg(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d", ctypes.c_int32), ("E", ctypes.c_int32),
                ("h", ctypes.c_int32), ("k", ctypes.c_int32), ("norm_topk", ctypes.c_int32),
                ("score", ctypes.c_int32), ("h_shared", ctypes.c_int32), ("dtype", ctypes.c_int32)]


def _ccfg(c: Cfg) -> _CCfg:
    return _CCfg(c.T, c.d, c.E, c.h, c.k, int(bool(c.norm_topk)),
                 SIGMOID if c.score == "sigmoid" else SOFTMAX, c.h_shared,
                 {"f32": F32, "f64": F64}.get(c.dtype, BF16))


def build(force: bool = False, source: str = _SRC, output: str = _LIB) -> str:
    """Compiles the C oracle into a shared library (plain gcc, IEEE double)."""
    if (not force and os.path.exists(output)
            and os.path.getmtime(output) >= os.path.getmtime(source)):
        return output
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall", "-Wextra",
           "-fno-fast-math", "-ffp-contract=off", source, "-o", output, "-lm"]
    subprocess.run(cmd, check=True)
    return output


_lib_cache: dict[str, ctypes.CDLL] = {}


def load(path: str | None = None) -> ctypes.CDLL:
    """Loads (building if needed) the oracle library; ``path`` selects another build."""
    if path is None:
        path = build()
    if path in _lib_cache:
        return _lib_cache[path]
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    lib.oracle_route.argtypes = [ctypes.POINTER(_CCfg), P, P, P, P, I64, I64, P, P, P, P, ctypes.c_int]
    lib.oracle_route.restype = ctypes.c_int
    lib.oracle_topk_margin.argtypes = [ctypes.POINTER(_CCfg), P, P, P, I64, I64, P, ctypes.c_int]
    lib.oracle_topk_margin.restype = ctypes.c_int
    lib.oracle_permute.argtypes = [ctypes.POINTER(_CCfg), P, P, P, P, P]
    lib.oracle_permute.restype = ctypes.c_int
    lib.oracle_forward.argtypes = [ctypes.POINTER(_CCfg), P, P, P, P, P, P, P, P, P, P, P, I64, P,
                                   ctypes.c_int]
    lib.oracle_forward.restype = ctypes.c_int
    lib.oracle_update_bias.argtypes = [ctypes.POINTER(_CCfg), P, ctypes.c_float, P, P]
    lib.oracle_update_bias.restype = ctypes.c_int
    lib.oracle_score_mean.argtypes = [ctypes.POINTER(_CCfg), P, P, P, ctypes.c_int]
    lib.oracle_score_mean.restype = ctypes.c_int
    lib.oracle_balance_loss.argtypes = [ctypes.POINTER(_CCfg), P, P, ctypes.c_double, P, P]
    lib.oracle_balance_loss.restype = ctypes.c_int
    lib.oracle_backward.argtypes = [ctypes.POINTER(_CCfg)] + [P] * 20 + [ctypes.c_int]
    lib.oracle_backward.restype = ctypes.c_int
    lib.oracle_quantize_q4.argtypes = [P, ctypes.c_int32, I64, ctypes.c_int32, P, P]
    lib.oracle_quantize_q4.restype = ctypes.c_int
    lib.oracle_dequantize_q4.argtypes = [P, P, I64, ctypes.c_int32, P]
    lib.oracle_dequantize_q4.restype = ctypes.c_int
    _lib_cache[path] = lib
    return lib


def _ptr(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _check_dtype(c: Cfg, *arrays):
    want = {"f32": np.float32, "f64": np.float64}.get(c.dtype, np.uint16)
    for a in arrays:
        if a is not None and a.dtype != want:
            raise TypeError(f"oracle expects {np.dtype(want)} arrays for dtype {c.dtype}, got {a.dtype}")


def _bias(c: Cfg, bias):
    """The balance bias as a C-contiguous float32 [E] array (or None)."""
    if bias is None:
        return None
    b = np.ascontiguousarray(bias, dtype=np.float32).reshape(-1)
    if b.size != c.E:
        raise ValueError(f"bias must have {c.E} entries, got {b.size}")
    return b


def route(c: Cfg, x, wr, w_sg=None, t0: int = 0, t1: int | None = None, want_probs=False,
          nthreads: int = 0, lib: ctypes.CDLL | None = None, bias=None):
    """Routes tokens [t0, t1).  Returns (ids[T,k] int32, gates[T,k], probs[T,E] | None,
    shared_gate[T] | None); rows outside [t0, t1) are left zero.  ``bias`` is the
    optional [E] float32 balance bias (selection only)."""
    lib = lib or load()
    _check_dtype(c, x, wr, w_sg)
    bias = _bias(c, bias)
    t1 = c.T if t1 is None else t1
    ids = np.zeros((c.T, c.k), np.int32)
    gates = np.zeros((c.T, c.k), np.float64)
    probs = np.zeros((c.T, c.E), np.float64) if want_probs else None
    sg = np.zeros((c.T,), np.float64) if (c.h_shared > 0 and w_sg is not None) else None
    cc = _ccfg(c)
    rc = lib.oracle_route(ctypes.byref(cc), _ptr(x), _ptr(wr), _ptr(w_sg), _ptr(bias), t0, t1,
                          _ptr(ids), _ptr(gates), _ptr(probs), _ptr(sg), nthreads)
    if rc != 0:
        raise ValueError("oracle_route rejected its arguments")
    return ids, gates, probs, sg


def topk_margin(c: Cfg, x, wr, t0: int = 0, t1: int | None = None, nthreads: int = 0,
                lib: ctypes.CDLL | None = None, bias=None):
    """Per-token smallest gap between adjacent keys among the top min(k+1, E)."""
    lib = lib or load()
    _check_dtype(c, x, wr)
    bias = _bias(c, bias)
    t1 = c.T if t1 is None else t1
    out = np.zeros((t1 - t0,), np.float64)
    cc = _ccfg(c)
    if lib.oracle_topk_margin(ctypes.byref(cc), _ptr(x), _ptr(wr), _ptr(bias), t0, t1, _ptr(out),
                              nthreads):
        raise ValueError("oracle_topk_margin rejected its arguments")
    return out


def permute(c: Cfg, ids, lib: ctypes.CDLL | None = None):
    """Returns (counts[E], offsets[E+1], sorted_rows[T*k], inv_rows[T*k]), all int32."""
    lib = lib or load()
    ids = np.ascontiguousarray(ids, dtype=np.int32).reshape(-1)
    R = c.T * c.k
    assert ids.size == R
    counts = np.zeros(c.E, np.int32)
    offsets = np.zeros(c.E + 1, np.int32)
    srt = np.zeros(R, np.int32)
    inv = np.zeros(R, np.int32)
    cc = _ccfg(c)
    if lib.oracle_permute(ctypes.byref(cc), _ptr(ids), _ptr(counts), _ptr(offsets), _ptr(srt),
                          _ptr(inv)):
        raise ValueError("oracle_permute rejected its arguments")
    return counts, offsets, srt, inv


def forward(c: Cfg, x, wr, wg, wu, wd, shared=None, tokens=None, nthreads: int = 0,
            lib: ctypes.CDLL | None = None, return_threads=False, bias=None):
    """Layer output rows (float64) for ``tokens`` (default: all).  ``shared`` is
    (W_shared_gate[h_s,d], W_shared_up[h_s,d], W_shared_down[d,h_s], w_s[d]) or None;
    ``bias`` the optional [E] float32 balance bias."""
    lib = lib or load()
    bias = _bias(c, bias)
    sh = shared if shared is not None else (None, None, None, None)
    _check_dtype(c, x, wr, wg, wu, wd, *sh)
    if tokens is None:
        tokens = np.arange(c.T, dtype=np.int64)
    tokens = np.ascontiguousarray(tokens, dtype=np.int64)
    y = np.zeros((tokens.size, c.d), np.float64)
    cc = _ccfg(c)
    rc = lib.oracle_forward(ctypes.byref(cc), _ptr(x), _ptr(wr), _ptr(wg), _ptr(wu), _ptr(wd),
                            _ptr(sh[0]), _ptr(sh[1]), _ptr(sh[2]), _ptr(sh[3]), _ptr(bias),
                            _ptr(tokens), tokens.size, _ptr(y), nthreads)
    if rc < 0:
        raise ValueError("oracle_forward rejected its arguments")
    return (y, rc) if return_threads else y


def update_bias(c: Cfg, counts, lr: float, bias, lib: ctypes.CDLL | None = None):
    """The balance bias after one step: bias + lr * sign(mean(counts) - counts), float32."""
    lib = lib or load()
    counts = np.ascontiguousarray(counts, dtype=np.int32).reshape(-1)
    assert counts.size == c.E
    b = _bias(c, bias)
    out = np.zeros(c.E, np.float32)
    if lib.oracle_update_bias(ctypes.byref(_ccfg(c)), _ptr(counts), ctypes.c_float(lr), _ptr(b), _ptr(out)):
        raise ValueError("oracle_update_bias rejected its arguments")
    return out


def score_mean(c: Cfg, x, wr, nthreads: int = 0, lib: ctypes.CDLL | None = None):
    """P_e: the mean over the T tokens of each expert's score (float64 [E])."""
    lib = lib or load()
    _check_dtype(c, x, wr)
    out = np.zeros(c.E, np.float64)
    if lib.oracle_score_mean(ctypes.byref(_ccfg(c)), _ptr(x), _ptr(wr), _ptr(out), nthreads):
        raise ValueError("oracle_score_mean rejected its arguments")
    return out


def balance_loss(c: Cfg, counts, score_mean_, alpha: float, lib: ctypes.CDLL | None = None):
    """(loss, f[E]): the Switch term alpha * E * sum_e f_e * P_e with f_e = counts[e] / T."""
    lib = lib or load()
    counts = np.ascontiguousarray(counts, dtype=np.int32).reshape(-1)
    pm = np.ascontiguousarray(score_mean_, dtype=np.float64).reshape(-1)
    assert counts.size == c.E and pm.size == c.E
    frac = np.zeros(c.E, np.float64)
    loss = np.zeros(1, np.float64)
    if lib.oracle_balance_loss(ctypes.byref(_ccfg(c)), _ptr(counts), _ptr(pm), ctypes.c_double(alpha),
                               _ptr(frac), _ptr(loss)):
        raise ValueError("oracle_balance_loss rejected its arguments")
    return float(loss[0]), frac


def backward(c: Cfg, x, wr, wg, wu, wd, dy, shared=None, bias=None, nthreads: int = 0,
             lib: ctypes.CDLL | None = None) -> dict:
    """Gradients (float64) of the layer given the upstream gradient dy[T, d] (the
    layer's dtype): dx, dw_router, dw_gate, dw_up, dw_down and, with a shared
    expert, dsh_gate, dsh_up, dsh_down, dw_shared_gate."""
    lib = lib or load()
    sh = shared if shared is not None else (None, None, None, None)
    _check_dtype(c, x, wr, wg, wu, wd, dy, *sh)
    bias = _bias(c, bias)
    g = {"dx": np.zeros((c.T, c.d)), "dw_router": np.zeros((c.E, c.d)), "dw_gate": np.zeros((c.E, c.h, c.d)),
         "dw_up": np.zeros((c.E, c.h, c.d)), "dw_down": np.zeros((c.E, c.d, c.h))}
    if c.h_shared > 0:
        g.update(dsh_gate=np.zeros((c.h_shared, c.d)), dsh_up=np.zeros((c.h_shared, c.d)),
                 dsh_down=np.zeros((c.d, c.h_shared)), dw_shared_gate=np.zeros(c.d))
    rc = lib.oracle_backward(ctypes.byref(_ccfg(c)), _ptr(x), _ptr(wr), _ptr(wg), _ptr(wu), _ptr(wd),
                             _ptr(sh[0]), _ptr(sh[1]), _ptr(sh[2]), _ptr(sh[3]), _ptr(bias), _ptr(dy),
                             _ptr(g["dx"]), _ptr(g["dw_router"]), _ptr(g["dw_gate"]), _ptr(g["dw_up"]),
                             _ptr(g["dw_down"]), _ptr(g.get("dsh_gate")), _ptr(g.get("dsh_up")),
                             _ptr(g.get("dsh_down")), _ptr(g.get("dw_shared_gate")), nthreads)
    if rc != 0:
        raise ValueError("oracle_backward rejected its arguments")
    return g


def quantize_q4(w, lib: ctypes.CDLL | None = None):
    """4-bit codes of a [..., cols] weight tensor (stored bits: uint16 bf16 or float32),
    cols a multiple of 64: (packed nibbles uint8 [..., cols / 2], scales float32
    [..., cols / 64])."""
    lib = lib or load()
    w = np.ascontiguousarray(w)
    dt = {np.dtype(np.uint16): BF16, np.dtype(np.float32): F32}[w.dtype]
    cols = w.shape[-1]
    rows = w.size // cols
    q = np.zeros(w.shape[:-1] + (cols // 2,), np.uint8)
    sc = np.zeros(w.shape[:-1] + (cols // 64,), np.float32)
    if lib.oracle_quantize_q4(_ptr(w), dt, rows, cols, _ptr(q), _ptr(sc)):
        raise ValueError("oracle_quantize_q4 rejected its arguments")
    return q, sc


def dequantize_q4(q, scales, lib: ctypes.CDLL | None = None):
    """The float64 values of a 4-bit tensor."""
    lib = lib or load()
    q = np.ascontiguousarray(q, np.uint8)
    scales = np.ascontiguousarray(scales, np.float32)
    cols = q.shape[-1] * 2
    rows = q.size // q.shape[-1]
    out = np.zeros(q.shape[:-1] + (cols,), np.float64)
    if lib.oracle_dequantize_q4(_ptr(q), _ptr(scales), rows, cols, _ptr(out)):
        raise ValueError("oracle_dequantize_q4 rejected its arguments")
    return out


def forward_q4(c: Cfg, x, wr, qg, sg_, qu, su, qd, sd, shared=None, tokens=None, bias=None, nthreads: int = 0,
               lib: ctypes.CDLL | None = None):
    """The layer with 4-bit routed experts: the routed weights are the values
    their codes represent, everything else as stored; evaluated by the float64
    forward on exact float64 copies of every input."""
    from . import dense
    f64 = Cfg(T=c.T, d=c.d, E=c.E, h=c.h, k=c.k, norm_topk=c.norm_topk, score=c.score, h_shared=c.h_shared,
              dtype="f64")
    sh = None
    if shared is not None:
        sh = tuple(np.ascontiguousarray(dense.to_f64(a)) for a in shared)
    return forward(f64, np.ascontiguousarray(dense.to_f64(x)), np.ascontiguousarray(dense.to_f64(wr)),
                   dequantize_q4(qg, sg_, lib), dequantize_q4(qu, su, lib), dequantize_q4(qd, sd, lib), sh,
                   tokens=tokens, bias=bias, nthreads=nthreads, lib=lib)
