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
            "moe_device_status", "moe_profile_events", "moe_launch_count", "moe_combine_noalloc", "moe_permute_workspace_size",
            "moe_selftest_wait_timeout",
            "moe_route_workspace_size"]
STAGES = ["route", "permute", "gate_up", "shared_gate_up", "down", "shared_down", "finalize"]


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({_status_string(status)})")


class MoEConfig(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d", ctypes.c_int32), ("E", ctypes.c_int32), ("h", ctypes.c_int32),
                ("k", ctypes.c_int32), ("norm_topk", ctypes.c_int32), ("score", ctypes.c_int32),
                ("h_shared", ctypes.c_int32), ("dtype", ctypes.c_int32)]


class WorkspaceViews(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("ids", "gates", "shared_gate", "counts", "offsets",
                                               "sorted_rows", "inv_rows", "act", "act_shared", "y_acc")]


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
            "moe_route": ([C, P, P, P, P, P, P, P, P, S, P], ctypes.c_int),
            "moe_route_workspace_size": ([C, ctypes.POINTER(S)], ctypes.c_int),
            "moe_permute": ([C, P, P, P, P, P, P, S, P], ctypes.c_int),
            "moe_permute_workspace_size": ([C, ctypes.POINTER(S)], ctypes.c_int),
            "moe_grouped_swiglu": ([C, P, P, P, P, P, P, P], ctypes.c_int),
            "moe_combine": ([C, P, P, P, P, P, P, P, S, P], ctypes.c_int),
            "moe_forward": ([C, P, P, P, P, P, P, P, P, P, P, P, S, P], ctypes.c_int),
            "moe_decode_max_rows": ([], ctypes.c_int32),
            "moe_device_status": ([P], ctypes.c_int),
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


def config(T, d, E, h, k, norm_topk=True, score="softmax", h_shared=0, dtype="bf16") -> MoEConfig:
    return MoEConfig(int(T), int(d), int(E), int(h), int(k), int(bool(norm_topk)),
                     1 if score == "sigmoid" else 0, int(h_shared), 1 if dtype == "f32" else 0)


def config_of(w: Workload, T: int | None = None) -> MoEConfig:
    return config(w.T if T is None else T, w.d, w.E, w.h, w.k, w.norm_topk, w.score, w.h_shared, w.dtype)


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
            "act_shared": ((T, cfg.h_shared), et), "y_acc": ((T, cfg.d), torch.float32)}
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


def route(cfg: MoEConfig, x, w_router, w_shared_gate=None, want_probs=False, ws=None, stream=None):
    """Returns (ids[T,k] int32, gates[T,k] f32, probs[T,E] | None, shared_gate[T] | None)."""
    et = _elem_dtype(cfg)
    dev = x.device
    if ws is None:
        n = route_workspace_size(cfg)
        ws = torch.empty(n, dtype=torch.uint8, device=dev) if n else None
    ids = torch.empty(cfg.T, cfg.k, dtype=torch.int32, device=dev)
    gates = torch.empty(cfg.T, cfg.k, dtype=torch.float32, device=dev)
    probs = torch.empty(cfg.T, cfg.E, dtype=torch.float32, device=dev) if want_probs else None
    sg = torch.empty(cfg.T, dtype=torch.float32, device=dev) if w_shared_gate is not None else None
    _check(lib().moe_route(ctypes.byref(cfg), _ptr(x, "x", (cfg.T, cfg.d), et),
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
    if ws is None and cfg.dtype == 0:
        ws = torch.empty(cfg.T * cfg.d * 4, dtype=torch.uint8, device=act.device)
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
            w_shared_gate=None, y=None, ws=None, stream=None):
    """The whole layer.  Returns y[T,d] (allocated unless given); ws is allocated if not given."""
    et = _elem_dtype(cfg)
    if y is None:
        y = torch.empty(cfg.T, cfg.d, dtype=et, device=x.device)
    if ws is None:
        ws = alloc_workspace(cfg, x.device)
    hs = cfg.h_shared
    _check(lib().moe_forward(ctypes.byref(cfg), _ptr(x, "x", (cfg.T, cfg.d), et),
                             _ptr(w_router, "w_router", (cfg.E, cfg.d), et),
                             _ptr(w_gate, "w_gate", (cfg.E, cfg.h, cfg.d), et),
                             _ptr(w_up, "w_up", (cfg.E, cfg.h, cfg.d), et),
                             _ptr(w_down, "w_down", (cfg.E, cfg.d, cfg.h), et),
                             _ptr(sh_gate, "sh_gate", (hs, cfg.d), et), _ptr(sh_up, "sh_up", (hs, cfg.d), et),
                             _ptr(sh_down, "sh_down", (cfg.d, hs), et),
                             _ptr(w_shared_gate, "w_shared_gate", (cfg.d,), et), _ptr(y, "y", (cfg.T, cfg.d), et),
                             _ptr(ws, "ws", dtype=torch.uint8), ws.numel(), _stream(stream)), "moe_forward")
    return y


def forward_layer(cfg: MoEConfig, layer, y=None, ws=None, stream=None):
    """moe_forward on a synth.Layer (device tensors)."""
    return forward(cfg, layer.x, layer.w_router, layer.w_gate, layer.w_up, layer.w_down, layer.sh_gate,
                   layer.sh_up, layer.sh_down, layer.w_shared_gate, y=y, ws=ws, stream=stream)


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
