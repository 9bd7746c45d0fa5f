"""Thin ctypes binding of libmoe.so (include/moe.h).

Argument marshalling only: every function checks shapes/dtypes/devices of the
torch tensors it is given, allocates outputs with torch (plumbing), and calls
the C entry point of the same name on the current CUDA stream.  No step of the
layer is computed here.  If libmoe.so is missing the first call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

from .workloads import Workload

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("MOE_LIB_PATH", os.path.join(_PKG, "libmoe.so"))

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
                4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE_TIMEOUT", 6: "MOE_ERR_DEVICE_INPUT"}
EXPORTED = ["moe_status_string", "moe_validate", "moe_workspace_size", "moe_workspace_layout", "moe_route",
            "moe_permute", "moe_grouped_swiglu", "moe_combine", "moe_forward", "moe_decode_max_rows",
            "moe_device_status", "moe_profile_events", "moe_profile_nvtx", "moe_launch_count", "moe_combine_noalloc", "moe_permute_workspace_size",
            "moe_selftest_wait_timeout",
            "moe_route_workspace_size", "moe_update_bias", "moe_balance_loss", "moe_train_workspace_size",
            "moe_forward_train", "moe_backward", "moe_quantize_q4", "moe_forward_q4",
            "moe_forward_host_workspace_size", "moe_forward_host"]
STAGES = ["route", "permute", "gate_up", "shared_gate_up", "down", "shared_down", "finalize"]


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({_status_string(status)})")


class MoEConfig(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d", ctypes.c_int32), ("E", ctypes.c_int32), ("h", ctypes.c_int32),
                ("k", ctypes.c_int32), ("norm_topk", ctypes.c_int32), ("score", ctypes.c_int32),
                ("h_shared", ctypes.c_int32), ("dtype", ctypes.c_int32), ("combine", ctypes.c_int32)]


class RouteOpts(ctypes.Structure):
    """moe_route_opts: balance bias (selection only) and the score-mean output."""
    _fields_ = [("balance_bias", ctypes.c_void_p), ("score_mean", ctypes.c_void_p)]


class WorkspaceViews(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("ids", "gates", "shared_gate", "counts", "offsets",
                                               "sorted_rows", "inv_rows", "act", "act_shared", "y_acc",
                                               "y_slots")]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m sparse_mixture_experts_sigmoid_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, S = ctypes.c_void_p, ctypes.c_size_t
        C = ctypes.POINTER(MoEConfig)
        sig = {
            "moe_status_string": ([ctypes.c_int], ctypes.c_char_p),
            "moe_validate": ([C], ctypes.c_int),
            "moe_workspace_size": ([C, ctypes.POINTER(S)], ctypes.c_int),
            "moe_workspace_layout": ([C, P, S, ctypes.POINTER(WorkspaceViews)], ctypes.c_int),
            "moe_route": ([C, ctypes.POINTER(RouteOpts), P, P, P, P, P, P, P, P, S, P], ctypes.c_int),
            "moe_route_workspace_size": ([C, ctypes.POINTER(S)], ctypes.c_int),
            "moe_permute": ([C, P, P, P, P, P, P, S, P], ctypes.c_int),
            "moe_permute_workspace_size": ([C, ctypes.POINTER(S)], ctypes.c_int),
            "moe_grouped_swiglu": ([C, P, P, P, P, P, P, P], ctypes.c_int),
            "moe_combine": ([C, P, P, P, P, P, P, P, S, P], ctypes.c_int),
            "moe_forward": ([C, ctypes.POINTER(RouteOpts), P, P, P, P, P, P, P, P, P, P, P, S, P],
                            ctypes.c_int),
            "moe_forward_host_workspace_size": ([C, ctypes.c_int32, ctypes.POINTER(S)], ctypes.c_int),
            "moe_forward_host": ([C] + [P] * 10 + [ctypes.c_int32, P, S, P, P], ctypes.c_int),
            "moe_update_bias": ([C, P, ctypes.c_float, P, P], ctypes.c_int),
            "moe_train_workspace_size": ([C, ctypes.POINTER(S)], ctypes.c_int),
            "moe_forward_train": ([C, ctypes.POINTER(RouteOpts), P, P, P, P, P, P, P, P, P, P, P, S, P],
                                  ctypes.c_int),
            "moe_backward": ([C] + [P] * 11 + [S] + [P] * 10, ctypes.c_int),
            "moe_quantize_q4": ([P, ctypes.c_int32, ctypes.c_int64, ctypes.c_int32, P, P, P], ctypes.c_int),
            "moe_forward_q4": ([C, ctypes.POINTER(RouteOpts)] + [P] * 13 + [P, S, P], ctypes.c_int),
            "moe_balance_loss": ([C, P, P, ctypes.c_float, P, P, P], ctypes.c_int),
            "moe_decode_max_rows": ([], ctypes.c_int32),
            "moe_device_status": ([P], ctypes.c_int),
            "moe_profile_nvtx": ([ctypes.c_int32], ctypes.c_int),
            "moe_selftest_wait_timeout": ([ctypes.c_uint32, P], ctypes.c_int),
            "moe_profile_events": ([ctypes.POINTER(ctypes.c_void_p), ctypes.c_int32], ctypes.c_int),
            "moe_launch_count": ([], ctypes.c_int64),
            "moe_combine_noalloc": ([C, P, P, P, P, P, P, P], ctypes.c_int),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes, f.restype = args, res
        _lib = L
    return _lib


def _status_string(s: int) -> str:
    try:
        return lib().moe_status_string(s).decode()
    except Exception:  # pragma: no cover - only used for messages
        return str(s)


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoEError(status, where)


COMBINE_MODES = {"add": 0, "ordered": 1}


def config(T, d, E, h, k, norm_topk=True, score="softmax", h_shared=0, dtype="bf16", combine="add") -> MoEConfig:
    """moe_config.  combine: "add" (fp32 reductions, summation order not fixed) or
    "ordered" (per-assignment slot rows added in slot order: bit-reproducible y)."""
    if combine not in COMBINE_MODES:
        raise ValueError(f"combine must be one of {sorted(COMBINE_MODES)}, got {combine!r}")
    return MoEConfig(int(T), int(d), int(E), int(h), int(k), int(bool(norm_topk)),
                     1 if score == "sigmoid" else 0, int(h_shared), 1 if dtype == "f32" else 0,
                     COMBINE_MODES[combine])


def config_of(w: Workload, T: int | None = None, combine: str = "add") -> MoEConfig:
    return config(w.T if T is None else T, w.d, w.E, w.h, w.k, w.norm_topk, w.score, w.h_shared, w.dtype,
                  combine)


def _elem_dtype(cfg: MoEConfig):
    return torch.float32 if cfg.dtype == 1 else torch.bfloat16


def _ptr(t: torch.Tensor | None, name: str, shape=None, dtype=None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def validate(cfg: MoEConfig) -> int:
    return lib().moe_validate(ctypes.byref(cfg))


def workspace_size(cfg: MoEConfig) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().moe_workspace_size(ctypes.byref(cfg), ctypes.byref(n)), "moe_workspace_size")
    return n.value


def alloc_workspace(cfg: MoEConfig, device=None) -> torch.Tensor:
    """A uint8 device tensor of moe_workspace_size bytes (torch allocations are 512-byte aligned)."""
    return torch.empty(max(workspace_size(cfg), 1), dtype=torch.uint8, device=device or "cuda")


def workspace_views(cfg: MoEConfig, ws: torch.Tensor) -> dict:
    """Torch views of the named workspace parts (after moe_forward they hold the routing)."""
    v = WorkspaceViews()
    _check(lib().moe_workspace_layout(ctypes.byref(cfg), _ptr(ws, "ws", dtype=torch.uint8),
                                      ws.numel(), ctypes.byref(v)), "moe_workspace_layout")
    base = ws.data_ptr()
    T, k, E, R = cfg.T, cfg.k, cfg.E, cfg.T * cfg.k
    et = _elem_dtype(cfg)
    spec = {"ids": ((T, k), torch.int32), "gates": ((T, k), torch.float32), "shared_gate": ((T,), torch.float32),
            "counts": ((E,), torch.int32), "offsets": ((E + 1,), torch.int32),
            "sorted_rows": ((R,), torch.int32), "inv_rows": ((R,), torch.int32), "act": ((R, cfg.h), et),
            "act_shared": ((T, cfg.h_shared), et), "y_acc": ((T, cfg.d), torch.float32),
            "y_slots": ((R, cfg.d), torch.float32)}
    out = {}
    for name, (shape, dt) in spec.items():
        p = getattr(v, name)
        if not p:
            out[name] = None
            continue
        off = p - base
        n = 1
        for s_ in shape:
            n *= s_
        nbytes = n * torch.empty((), dtype=dt).element_size()
        out[name] = ws[off:off + nbytes].view(dt).view(shape)
    return out


def route_workspace_size(cfg: MoEConfig) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().moe_route_workspace_size(ctypes.byref(cfg), ctypes.byref(n)), "moe_route_workspace_size")
    return n.value


def route_opts(cfg: MoEConfig, balance_bias=None, score_mean=None):
    """A moe_route_opts for ctypes (None when both are absent).  balance_bias and
    score_mean are [E] float32 CUDA tensors (score_mean is written)."""
    if balance_bias is None and score_mean is None:
        return None
    return ctypes.byref(RouteOpts(_ptr(balance_bias, "balance_bias", (cfg.E,), torch.float32),
                                  _ptr(score_mean, "score_mean", (cfg.E,), torch.float32)))


def route(cfg: MoEConfig, x, w_router, w_shared_gate=None, want_probs=False, ws=None, stream=None,
          balance_bias=None, score_mean=None):
    """Returns (ids[T,k] int32, gates[T,k] f32, probs[T,E] | None, shared_gate[T] | None).
    balance_bias: optional [E] float32 selection bias; score_mean: optional [E]
    float32 tensor that receives the mean score per expert."""
    et = _elem_dtype(cfg)
    dev = x.device
    if ws is None:
        n = route_workspace_size(cfg)
        ws = torch.empty(n, dtype=torch.uint8, device=dev) if n else None
    ids = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=dev)
    gates = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device=dev)
    probs = torch.empty(cfg.T, cfg.E, dtype=torch.float32, device=dev) if want_probs else None
    sg = torch.empty(cfg.T, dtype=torch.float32, device=dev) if w_shared_gate is not None else None
    _check(lib().moe_route(ctypes.byref(cfg), route_opts(cfg, balance_bias, score_mean),
                           _ptr(x, "x", (cfg.T, cfg.d), et),
                           _ptr(w_router, "w_router", (cfg.E, cfg.d), et),
                           _ptr(w_shared_gate, "w_shared_gate", (cfg.d,), et), _ptr(ids, "ids"),
                           _ptr(gates, "gates"), _ptr(probs, "probs"), _ptr(sg, "shared_gate"), _ptr(ws, "ws"),
                           0 if ws is None else ws.numel() * ws.element_size(), _stream(stream)),
           "moe_route")
    return ids, gates, probs, sg


def permute_workspace_size(cfg: MoEConfig) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().moe_permute_workspace_size(ctypes.byref(cfg), ctypes.byref(n)), "moe_permute_workspace_size")
    return n.value


def permute(cfg: MoEConfig, ids, ws=None, stream=None):
    """Returns (counts[E], offsets[E+1], sorted_rows[T*k], inv_rows[T*k]), int32."""
    dev = ids.device
    if ws is None:
        ws = torch.empty(max(permute_workspace_size(cfg), 16), dtype=torch.uint8, device=dev)
    R = cfg.T * cfg.k
    counts = torch.empty(cfg.E, dtype=torch.int32, device=dev)
    offsets = torch.empty(cfg.E + 1, dtype=torch.int32, device=dev)
    srt = torch.empty(max(R, 1), dtype=torch.int32, device=dev)[:R]
    inv = torch.empty(max(R, 1), dtype=torch.int32, device=dev)[:R]
    _check(lib().moe_permute(ctypes.byref(cfg), _ptr(ids, "ids", (cfg.T, cfg.k), torch.int32),
                             _ptr(counts, "counts"), _ptr(offsets, "offsets"), _ptr(srt, "sorted_rows"),
                             _ptr(inv, "inv_rows"), _ptr(ws, "ws"), ws.numel() * ws.element_size(),
                             _stream(stream)), "moe_permute")
    return counts, offsets, srt, inv


def grouped_swiglu(cfg: MoEConfig, x, w_gate, w_up, offsets, sorted_rows, stream=None):
    et = _elem_dtype(cfg)
    act = torch.empty(cfg.T * cfg.k, cfg.h, dtype=et, device=x.device)
    _check(lib().moe_grouped_swiglu(ctypes.byref(cfg), _ptr(x, "x", (cfg.T, cfg.d), et),
                                    _ptr(w_gate, "w_gate", (cfg.E, cfg.h, cfg.d), et),
                                    _ptr(w_up, "w_up", (cfg.E, cfg.h, cfg.d), et),
                                    _ptr(offsets, "offsets", (cfg.E + 1,), torch.int32),
                                    _ptr(sorted_rows, "sorted_rows", (cfg.T * cfg.k,), torch.int32),
                                    _ptr(act, "act"), _stream(stream)), "moe_grouped_swiglu")
    return act


def combine(cfg: MoEConfig, act, w_down, offsets, sorted_rows, gates, ws=None, stream=None):
    et = _elem_dtype(cfg)
    y = torch.empty(cfg.T, cfg.d, dtype=et, device=act.device)
    if ws is None and (cfg.dtype == 0 or cfg.combine == COMBINE_MODES["ordered"]):
        # the fp32 accumulator [T, d], or the ordered combine's slot rows [T*k, d]
        rows = cfg.T * cfg.k if cfg.combine == COMBINE_MODES["ordered"] else cfg.T
        ws = torch.empty(rows * cfg.d * 4, dtype=torch.uint8, device=act.device)
    _check(lib().moe_combine(ctypes.byref(cfg), _ptr(act, "act", (cfg.T * cfg.k, cfg.h), et),
                             _ptr(w_down, "w_down", (cfg.E, cfg.d, cfg.h), et),
                             _ptr(offsets, "offsets", (cfg.E + 1,), torch.int32),
                             _ptr(sorted_rows, "sorted_rows", (cfg.T * cfg.k,), torch.int32),
                             _ptr(gates, "gates", (cfg.T, cfg.k), torch.float32), _ptr(y, "y"),
                             _ptr(ws, "ws"), 0 if ws is None else ws.numel() * ws.element_size(),
                             _stream(stream)), "moe_combine")
    return y


def combine_noalloc(cfg: MoEConfig, act, w_down, offsets, sorted_rows, gates, y=None, stream=None):
    """moe_combine_noalloc: like combine() but the library's static accumulator
    replaces the workspace (for callers that cannot allocate device memory)."""
    et = _elem_dtype(cfg)
    if y is None:
        y = torch.empty(cfg.T, cfg.d, dtype=et, device=act.device)
    _check(lib().moe_combine_noalloc(ctypes.byref(cfg), _ptr(act, "act", (cfg.T * cfg.k, cfg.h), et),
                                     _ptr(w_down, "w_down", (cfg.E, cfg.d, cfg.h), et),
                                     _ptr(offsets, "offsets", (cfg.E + 1,), torch.int32),
                                     _ptr(sorted_rows, "sorted_rows", (cfg.T * cfg.k,), torch.int32),
                                     _ptr(gates, "gates", (cfg.T, cfg.k), torch.float32),
                                     _ptr(y, "y", (cfg.T, cfg.d), et), _stream(stream)), "moe_combine_noalloc")
    return y


def forward(cfg: MoEConfig, x, w_router, w_gate, w_up, w_down, sh_gate=None, sh_up=None, sh_down=None,
            w_shared_gate=None, y=None, ws=None, stream=None, balance_bias=None, score_mean=None):
    """The whole layer.  Returns y[T,d] (allocated unless given); ws is allocated if not given.
    balance_bias / score_mean: the routing options (see route())."""
    et = _elem_dtype(cfg)
    if y is None:
        y = torch.empty(cfg.T, cfg.d, dtype=et, device=x.device)
    if ws is None:
        ws = alloc_workspace(cfg, x.device)
    hs = cfg.h_shared
    _check(lib().moe_forward(ctypes.byref(cfg), route_opts(cfg, balance_bias, score_mean),
                             _ptr(x, "x", (cfg.T, cfg.d), et),
                             _ptr(w_router, "w_router", (cfg.E, cfg.d), et),
                             _ptr(w_gate, "w_gate", (cfg.E, cfg.h, cfg.d), et),
                             _ptr(w_up, "w_up", (cfg.E, cfg.h, cfg.d), et),
                             _ptr(w_down, "w_down", (cfg.E, cfg.d, cfg.h), et),
                             _ptr(sh_gate, "sh_gate", (hs, cfg.d), et), _ptr(sh_up, "sh_up", (hs, cfg.d), et),
                             _ptr(sh_down, "sh_down", (cfg.d, hs), et),
                             _ptr(w_shared_gate, "w_shared_gate", (cfg.d,), et), _ptr(y, "y", (cfg.T, cfg.d), et),
                             _ptr(ws, "ws", dtype=torch.uint8), ws.numel(), _stream(stream)), "moe_forward")
    return y


def forward_layer(cfg: MoEConfig, layer, y=None, ws=None, stream=None, balance_bias=None, score_mean=None):
    """moe_forward on a synth.Layer (device tensors)."""
    return forward(cfg, layer.x, layer.w_router, layer.w_gate, layer.w_up, layer.w_down, layer.sh_gate,
                   layer.sh_up, layer.sh_down, layer.w_shared_gate, y=y, ws=ws, stream=stream,
                   balance_bias=balance_bias, score_mean=score_mean)


def _host_ptr(t: torch.Tensor, name: str, shape, dtype):
    if t.is_cuda:
        raise ValueError(f"{name} must be a host tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.dtype != dtype or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must be {dtype} of shape {tuple(shape)}")
    return ctypes.c_void_p(t.data_ptr())


def host_piece_bounds(T: int, chunks: int) -> list[int]:
    """The token bounds of moe_forward_host's pieces (its documented rule: n = min(chunks, T, 256);
    with n >= 3 the first and last pieces are half as large as the others)."""
    n = min(chunks, T, 256)
    if n <= 0:
        return [0]
    if n <= 2:
        return [T * i // n for i in range(n + 1)]
    c = [0] + [2 * i - 1 for i in range(1, n)] + [2 * n - 2]
    return [T * ci // (2 * n - 2) for ci in c]


def forward_host_workspace_size(cfg: MoEConfig, chunks: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().moe_forward_host_workspace_size(ctypes.byref(cfg), int(chunks), ctypes.byref(n)),
           "moe_forward_host_workspace_size")
    return n.value


def forward_host(cfg: MoEConfig, layer, x_host, y_host, chunks: int, ws=None, stream=None, copy_stream=None):
    """moe_forward_host: x_host [T,d] in and y_host [T,d] out in (pinned) host memory, the weights of
    the synth.Layer-like `layer` on the device; `chunks` pieces whose copies overlap the other pieces'
    layers (copy_stream: a torch.cuda.Stream, or None for no overlap).  Returns y_host."""
    et = _elem_dtype(cfg)
    if ws is None:
        ws = torch.empty(max(forward_host_workspace_size(cfg, chunks), 1), dtype=torch.uint8, device="cuda")
    hs = cfg.h_shared
    cs = ctypes.c_void_p(copy_stream.cuda_stream) if copy_stream is not None else None
    _check(lib().moe_forward_host(ctypes.byref(cfg), _host_ptr(x_host, "x_host", (cfg.T, cfg.d), et),
                                  _ptr(layer.w_router, "w_router", (cfg.E, cfg.d), et),
                                  _ptr(layer.w_gate, "w_gate", (cfg.E, cfg.h, cfg.d), et),
                                  _ptr(layer.w_up, "w_up", (cfg.E, cfg.h, cfg.d), et),
                                  _ptr(layer.w_down, "w_down", (cfg.E, cfg.d, cfg.h), et),
                                  _ptr(layer.sh_gate, "sh_gate", (hs, cfg.d), et),
                                  _ptr(layer.sh_up, "sh_up", (hs, cfg.d), et),
                                  _ptr(layer.sh_down, "sh_down", (cfg.d, hs), et),
                                  _ptr(layer.w_shared_gate, "w_shared_gate", (cfg.d,), et),
                                  _host_ptr(y_host, "y_host", (cfg.T, cfg.d), et), int(chunks),
                                  _ptr(ws, "ws", dtype=torch.uint8), ws.numel(), _stream(stream), cs),
           "moe_forward_host")
    return y_host


def update_bias(cfg: MoEConfig, counts, lr: float, bias, stream=None):
    """moe_update_bias: bias[E] (float32, in place) += lr * sign(mean(counts) - counts)."""
    _check(lib().moe_update_bias(ctypes.byref(cfg), _ptr(counts, "counts", (cfg.E,), torch.int32),
                                 ctypes.c_float(lr), _ptr(bias, "bias", (cfg.E,), torch.float32),
                                 _stream(stream)), "moe_update_bias")
    return bias


def balance_loss(cfg: MoEConfig, counts, score_mean, alpha: float, want_frac=False, stream=None):
    """moe_balance_loss: returns (loss[1] float32, f[E] float32 | None) on the device."""
    dev = counts.device
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    frac = torch.empty(cfg.E, dtype=torch.float32, device=dev) if want_frac else None
    _check(lib().moe_balance_loss(ctypes.byref(cfg), _ptr(counts, "counts", (cfg.E,), torch.int32),
                                  _ptr(score_mean, "score_mean", (cfg.E,), torch.float32),
                                  ctypes.c_float(alpha), _ptr(frac, "frac"), _ptr(loss, "loss"),
                                  _stream(stream)), "moe_balance_loss")
    return loss, frac


def device_status(stream=None) -> int:
    return lib().moe_device_status(_stream(stream))


def decode_max_rows() -> int:
    return lib().moe_decode_max_rows()


def selftest_wait_timeout(limit_ms: int, stream=None) -> int:
    """Enqueues the bounded-wait self-test kernel (see moe_selftest_wait_timeout);
    returns the launch status (the timeout itself shows in device_status())."""
    return lib().moe_selftest_wait_timeout(int(limit_ms), _stream(stream))


def launch_count() -> int:
    """Kernels launched by libmoe.so so far in this process."""
    return lib().moe_launch_count()


class StageEvents:
    """CUDA events that moe_forward records between its stages (moe_profile_events)."""

    def __init__(self):
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(len(STAGES) + 1)]
        for e in self.events:
            e.record()          # materialise the cudaEvent_t handles
        torch.cuda.synchronize()
        self._arr = (ctypes.c_void_p * len(self.events))(*[e.cuda_event for e in self.events])

    def __enter__(self):
        _check(lib().moe_profile_events(self._arr, len(self.events)), "moe_profile_events")
        return self

    def __exit__(self, *exc):
        lib().moe_profile_events(None, 0)

    def stage_ms(self) -> dict:
        """Per-stage milliseconds of the last recorded moe_forward (call after a synchronize)."""
        return {n: self.events[i].elapsed_time(self.events[i + 1]) for i, n in enumerate(STAGES)}


# ----------------------------------------------------------------------------- training

def train_workspace_size(cfg: MoEConfig) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().moe_train_workspace_size(ctypes.byref(cfg), ctypes.byref(n)), "moe_train_workspace_size")
    return n.value


def alloc_train_workspace(cfg: MoEConfig, device=None) -> torch.Tensor:
    """A uint8 device tensor of moe_train_workspace_size bytes."""
    return torch.empty(max(train_workspace_size(cfg), 1), dtype=torch.uint8, device=device or "cuda")


def forward_train(cfg: MoEConfig, layer, ws, y=None, stream=None, balance_bias=None, score_mean=None):
    """moe_forward_train on a synth.Layer: y[T,d]; ws (alloc_train_workspace) keeps what
    backward() needs."""
    et = _elem_dtype(cfg)
    if y is None:
        y = torch.empty(cfg.T, cfg.d, dtype=et, device=layer.x.device)
    hs = cfg.h_shared
    _check(lib().moe_forward_train(ctypes.byref(cfg), route_opts(cfg, balance_bias, score_mean),
                                   _ptr(layer.x, "x", (cfg.T, cfg.d), et),
                                   _ptr(layer.w_router, "w_router", (cfg.E, cfg.d), et),
                                   _ptr(layer.w_gate, "w_gate", (cfg.E, cfg.h, cfg.d), et),
                                   _ptr(layer.w_up, "w_up", (cfg.E, cfg.h, cfg.d), et),
                                   _ptr(layer.w_down, "w_down", (cfg.E, cfg.d, cfg.h), et),
                                   _ptr(layer.sh_gate, "sh_gate", (hs, cfg.d), et),
                                   _ptr(layer.sh_up, "sh_up", (hs, cfg.d), et),
                                   _ptr(layer.sh_down, "sh_down", (cfg.d, hs), et),
                                   _ptr(layer.w_shared_gate, "w_shared_gate", (cfg.d,), et),
                                   _ptr(y, "y", (cfg.T, cfg.d), et), _ptr(ws, "ws", dtype=torch.uint8), ws.numel(),
                                   _stream(stream)), "moe_forward_train")
    return y


def backward(cfg: MoEConfig, layer, dy, ws, grads=None, stream=None) -> dict:
    """moe_backward after forward_train(cfg, layer, ws): the gradients (allocated
    unless ``grads`` holds them) dx, dw_router (fp32), dw_gate, dw_up, dw_down and,
    with a shared expert, dsh_gate, dsh_up, dsh_down, dw_shared_gate (fp32)."""
    et = _elem_dtype(cfg)
    dev = layer.x.device
    hs = cfg.h_shared
    if grads is None:
        grads = {"dx": torch.empty(cfg.T, cfg.d, dtype=et, device=dev),
                 "dw_router": torch.empty(cfg.E, cfg.d, dtype=torch.float32, device=dev),
                 "dw_gate": torch.empty(cfg.E, cfg.h, cfg.d, dtype=et, device=dev),
                 "dw_up": torch.empty(cfg.E, cfg.h, cfg.d, dtype=et, device=dev),
                 "dw_down": torch.empty(cfg.E, cfg.d, cfg.h, dtype=et, device=dev)}
        if hs:
            grads.update(dsh_gate=torch.empty(hs, cfg.d, dtype=et, device=dev),
                         dsh_up=torch.empty(hs, cfg.d, dtype=et, device=dev),
                         dsh_down=torch.empty(cfg.d, hs, dtype=et, device=dev),
                         dw_shared_gate=torch.empty(cfg.d, dtype=torch.float32, device=dev))
    g = grads
    _check(lib().moe_backward(ctypes.byref(cfg), _ptr(layer.x, "x", (cfg.T, cfg.d), et),
                              _ptr(layer.w_router, "w_router", (cfg.E, cfg.d), et),
                              _ptr(layer.w_gate, "w_gate", (cfg.E, cfg.h, cfg.d), et),
                              _ptr(layer.w_up, "w_up", (cfg.E, cfg.h, cfg.d), et),
                              _ptr(layer.w_down, "w_down", (cfg.E, cfg.d, cfg.h), et),
                              _ptr(layer.sh_gate, "sh_gate", (hs, cfg.d), et),
                              _ptr(layer.sh_up, "sh_up", (hs, cfg.d), et),
                              _ptr(layer.sh_down, "sh_down", (cfg.d, hs), et),
                              _ptr(layer.w_shared_gate, "w_shared_gate", (cfg.d,), et),
                              _ptr(dy, "dy", (cfg.T, cfg.d), et), _ptr(ws, "ws", dtype=torch.uint8), ws.numel(),
                              _ptr(g["dx"], "dx", (cfg.T, cfg.d), et),
                              _ptr(g["dw_router"], "dw_router", (cfg.E, cfg.d), torch.float32),
                              _ptr(g["dw_gate"], "dw_gate", (cfg.E, cfg.h, cfg.d), et),
                              _ptr(g["dw_up"], "dw_up", (cfg.E, cfg.h, cfg.d), et),
                              _ptr(g["dw_down"], "dw_down", (cfg.E, cfg.d, cfg.h), et),
                              _ptr(g.get("dsh_gate"), "dsh_gate", (hs, cfg.d), et),
                              _ptr(g.get("dsh_up"), "dsh_up", (hs, cfg.d), et),
                              _ptr(g.get("dsh_down"), "dsh_down", (cfg.d, hs), et),
                              _ptr(g.get("dw_shared_gate"), "dw_shared_gate", (cfg.d,), torch.float32),
                              _stream(stream)), "moe_backward")
    return grads


# ----------------------------------------------------------------------------- 4-bit routed experts

def quantize_q4(w: torch.Tensor, stream=None):
    """moe_quantize_q4 of a [..., cols] bf16/fp32 CUDA tensor: (codes uint8
    [..., cols / 2], scales float32 [..., cols / 64])."""
    cols = w.shape[-1]
    rows = w.numel() // cols
    q = torch.empty(*w.shape[:-1], cols // 2, dtype=torch.uint8, device=w.device)
    sc = torch.empty(*w.shape[:-1], cols // 64, dtype=torch.float32, device=w.device)
    _check(lib().moe_quantize_q4(_ptr(w, "w"), 1 if w.dtype == torch.float32 else 0, rows, cols, _ptr(q, "q"),
                                 _ptr(sc, "scales"), _stream(stream)), "moe_quantize_q4")
    return q, sc


def quantize_experts_q4(layer, stream=None) -> dict:
    """The routed experts of a synth.Layer in 4 bits: {"q_gate", "s_gate", "q_up", "s_up", "q_down", "s_down"}."""
    out = {}
    for name, w in (("gate", layer.w_gate), ("up", layer.w_up), ("down", layer.w_down)):
        out["q_" + name], out["s_" + name] = quantize_q4(w, stream)
    return out


def forward_q4(cfg: MoEConfig, layer, q4: dict, y=None, ws=None, stream=None, balance_bias=None, score_mean=None):
    """moe_forward_q4: the layer with 4-bit routed experts (q4 from quantize_experts_q4)."""
    et = _elem_dtype(cfg)
    if y is None:
        y = torch.empty(cfg.T, cfg.d, dtype=et, device=layer.x.device)
    if ws is None:
        ws = alloc_workspace(cfg, layer.x.device)
    hs = cfg.h_shared
    E, h, d = cfg.E, cfg.h, cfg.d
    _check(lib().moe_forward_q4(ctypes.byref(cfg), route_opts(cfg, balance_bias, score_mean),
                                _ptr(layer.x, "x", (cfg.T, d), et), _ptr(layer.w_router, "w_router", (E, d), et),
                                _ptr(q4["q_gate"], "q_gate", (E, h, d // 2), torch.uint8),
                                _ptr(q4["s_gate"], "s_gate", (E, h, d // 64), torch.float32),
                                _ptr(q4["q_up"], "q_up", (E, h, d // 2), torch.uint8),
                                _ptr(q4["s_up"], "s_up", (E, h, d // 64), torch.float32),
                                _ptr(q4["q_down"], "q_down", (E, d, h // 2), torch.uint8),
                                _ptr(q4["s_down"], "s_down", (E, d, h // 64), torch.float32),
                                _ptr(layer.sh_gate, "sh_gate", (hs, d), et), _ptr(layer.sh_up, "sh_up", (hs, d), et),
                                _ptr(layer.sh_down, "sh_down", (d, hs), et),
                                _ptr(layer.w_shared_gate, "w_shared_gate", (d,), et), _ptr(y, "y", (cfg.T, d), et),
                                _ptr(ws, "ws", dtype=torch.uint8), ws.numel(), _stream(stream)), "moe_forward_q4")
    return y


def profile_nvtx(on: bool = True) -> None:
    """moe_profile_nvtx: NVTX ranges around each forward stage on this thread."""
    _check(lib().moe_profile_nvtx(int(bool(on))), "moe_profile_nvtx")

