"""ctypes binding of libdora.so (include/dora.h), same names as the C ABI.

Argument marshalling only: torch tensors are checked (device, dtype,
contiguity), their data pointers, sizes and the current CUDA stream are
passed to the library, and a non-OK status raises ``DoraError``.  Outputs and
workspaces that the caller does not pass are allocated with torch (device
memory plumbing); every step of the computation runs in the library's CUDA
kernels.  There is no fallback: if libdora.so cannot be loaded, every call
raises.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Sequence

import torch

from . import build as _build

DORA_OK, DORA_ERR_INVALID_ARG, DORA_ERR_UNSUPPORTED, DORA_ERR_WORKSPACE, DORA_ERR_CUDA, \
    DORA_ERR_TIMEOUT, DORA_ERR_BOUNDS, DORA_ERR_INTERNAL = range(8)
DORA_F32, DORA_BF16 = 0, 1
DORA_MAX_RANK = 512
DORA_MAX_GROUP = 1024
DORA_MAX_COMPOSE_GROUP = 64

# Symbols include/dora.h declares (the ABI test checks the library exports each).
EXPORTED = (
    "dora_factored_norm_workspace_size", "dora_factored_norm",
    "dora_factored_norm_grouped_workspace_size", "dora_factored_norm_grouped",
    "dora_compose_fwd", "dora_compose_bwd_workspace_size", "dora_compose_bwd",
    "dora_get_device_status", "dora_status_string", "dora_version", "dora_launch_count",
    "dora_set_wait_timeout_ns", "dora_debug_unsignalled_wait", "dora_set_timing_events",
    "dora_last_error", "dora_set_trace_buffer", "dora_compose_bwd_static",
    "dora_compose_fwd_train", "dora_compose_bwd_inner", "dora_compose_bwd_frozen",
    "dora_compose_fwd_grouped", "dora_compose_bwd_grouped_workspace_size",
    "dora_compose_bwd_grouped", "dora_merge_weight_workspace_size", "dora_merge_weight",
    "dora_factored_norm_sq", "dora_norm_finalize", "dora_compose_fwd_delta",
    "dora_norm_plan_check",
)


class DoraError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = ""
        if status in (DORA_ERR_CUDA, DORA_ERR_INTERNAL):
            detail = " [" + load_library().dora_last_error().decode() + "]"
        super().__init__(f"{where}: {status_string(status)} (status {status}){detail}")


class NormProblem(ctypes.Structure):
    _fields_ = [
        ("W0", ctypes.c_void_p), ("A", ctypes.c_void_p), ("B", ctypes.c_void_p),
        ("m", ctypes.c_void_p), ("n_out", ctypes.c_void_p), ("g_out", ctypes.c_void_p),
        ("d_out", ctypes.c_int64), ("d_in", ctypes.c_int64), ("r", ctypes.c_int64),
        ("s", ctypes.c_float),
    ]


class ComposeProblem(ctypes.Structure):
    _fields_ = [
        ("base", ctypes.c_void_p), ("lora", ctypes.c_void_p), ("inner", ctypes.c_void_p),
        ("m", ctypes.c_void_p), ("n", ctypes.c_void_p), ("y", ctypes.c_void_p),
        ("dy", ctypes.c_void_p), ("d_base", ctypes.c_void_p), ("d_lora", ctypes.c_void_p),
        ("dm", ctypes.c_void_p), ("T", ctypes.c_int64), ("d_out", ctypes.c_int64),
        ("s", ctypes.c_float),
    ]


_lib = None
_lock = threading.Lock()


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Loads libdora.so (built in-tree); raises if it is missing."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = path or _build.library_path()
        if not os.path.exists(path):
            raise RuntimeError(
                f"{path} is missing: build it with `python -m dora_adapter_factored_b200.build`")
        lib = ctypes.CDLL(path)
        c_i64, c_sz, c_vp, c_f, c_i = (ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p,
                                       ctypes.c_float, ctypes.c_int)
        lib.dora_factored_norm_workspace_size.argtypes = [c_i64, c_i64, c_i64, c_i]
        lib.dora_factored_norm_workspace_size.restype = c_sz
        lib.dora_factored_norm.argtypes = [c_vp, c_vp, c_vp, c_i, c_i64, c_i64, c_i64, c_f, c_vp,
                                           c_f, c_vp, c_vp, c_vp, c_sz, c_vp]
        lib.dora_factored_norm.restype = c_i
        lib.dora_factored_norm_grouped_workspace_size.argtypes = [ctypes.POINTER(NormProblem),
                                                                  c_i, c_i]
        lib.dora_factored_norm_grouped_workspace_size.restype = c_sz
        lib.dora_factored_norm_grouped.argtypes = [ctypes.POINTER(NormProblem), c_i, c_i, c_f,
                                                   c_vp, c_sz, c_vp]
        lib.dora_factored_norm_grouped.restype = c_i
        lib.dora_compose_fwd.argtypes = [c_vp, c_vp, c_vp, c_vp, c_f, c_f, c_i, c_i64, c_i64, c_vp,
                                         c_vp]
        lib.dora_compose_fwd.restype = c_i
        lib.dora_compose_fwd_delta.argtypes = [c_vp, c_vp, c_vp, c_vp, c_f, c_f, c_i, c_i64, c_i64,
                                               c_vp, c_vp]
        lib.dora_compose_fwd_delta.restype = c_i
        lib.dora_compose_bwd_workspace_size.argtypes = [c_i64, c_i64, c_i]
        lib.dora_compose_bwd_workspace_size.restype = c_sz
        lib.dora_compose_bwd.argtypes = [c_vp, c_vp, c_vp, c_vp, c_vp, c_f, c_f, c_i, c_i64, c_i64,
                                         c_vp, c_vp, c_vp, c_vp, c_sz, c_vp]
        lib.dora_compose_bwd.restype = c_i
        lib.dora_get_device_status.argtypes = [c_vp]
        lib.dora_get_device_status.restype = c_i
        lib.dora_status_string.argtypes = [c_i]
        lib.dora_status_string.restype = ctypes.c_char_p
        lib.dora_version.argtypes = []
        lib.dora_version.restype = c_i
        lib.dora_launch_count.argtypes = []
        lib.dora_launch_count.restype = ctypes.c_uint64
        lib.dora_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
        lib.dora_set_wait_timeout_ns.restype = None
        lib.dora_debug_unsignalled_wait.argtypes = [ctypes.c_uint64, c_vp]
        lib.dora_debug_unsignalled_wait.restype = c_i
        lib.dora_set_timing_events.argtypes = [c_vp, c_vp]
        lib.dora_set_timing_events.restype = None
        lib.dora_last_error.argtypes = []
        lib.dora_last_error.restype = ctypes.c_char_p
        lib.dora_set_trace_buffer.argtypes = [c_vp]
        lib.dora_set_trace_buffer.restype = None
        lib.dora_norm_plan_check.argtypes = [ctypes.POINTER(c_i64)] * 3 + [c_i, c_i, c_i]
        lib.dora_norm_plan_check.restype = c_i
        lib.dora_compose_bwd_static.argtypes = [c_vp, c_vp, c_vp, c_vp, c_vp, c_f, c_f, c_i,
                                                c_i64, c_i64, c_vp, c_vp, c_vp, c_vp]
        lib.dora_compose_bwd_static.restype = c_i
        lib.dora_compose_fwd_train.argtypes = [c_vp, c_vp, c_vp, c_vp, c_f, c_f, c_i, c_i64, c_i64,
                                               c_vp, c_vp, c_vp]
        lib.dora_compose_fwd_train.restype = c_i
        lib.dora_compose_bwd_inner.argtypes = [c_vp, c_vp, c_vp, c_vp, c_f, c_f, c_i, c_i64, c_i64,
                                               c_vp, c_vp, c_vp, c_vp, c_sz, c_vp]
        lib.dora_compose_bwd_inner.restype = c_i
        lib.dora_compose_bwd_frozen.argtypes = [c_vp, c_vp, c_vp, c_f, c_f, c_i, c_i64, c_i64,
                                                c_vp, c_vp, c_vp]
        lib.dora_compose_bwd_frozen.restype = c_i
        cp = ctypes.POINTER(ComposeProblem)
        lib.dora_compose_fwd_grouped.argtypes = [cp, c_i, c_i, c_f, c_vp]
        lib.dora_compose_fwd_grouped.restype = c_i
        lib.dora_compose_bwd_grouped_workspace_size.argtypes = [cp, c_i, c_i]
        lib.dora_compose_bwd_grouped_workspace_size.restype = c_sz
        lib.dora_compose_bwd_grouped.argtypes = [cp, c_i, c_i, c_f, c_vp, c_sz, c_vp]
        lib.dora_compose_bwd_grouped.restype = c_i
        lib.dora_merge_weight_workspace_size.argtypes = [c_i64, c_i64, c_i64]
        lib.dora_merge_weight_workspace_size.restype = c_sz
        lib.dora_merge_weight.argtypes = [c_vp, c_vp, c_vp, c_vp, c_vp, c_f, c_f, c_i64, c_i64,
                                          c_i64, c_vp, c_vp, c_sz, c_vp]
        lib.dora_merge_weight.restype = c_i
        lib.dora_factored_norm_sq.argtypes = [c_vp, c_vp, c_vp, c_i, c_i64, c_i64, c_i64, c_f,
                                              c_vp, c_vp, c_sz, c_vp]
        lib.dora_factored_norm_sq.restype = c_i
        lib.dora_norm_finalize.argtypes = [c_vp, c_vp, c_f, c_i64, c_vp, c_vp, c_vp]
        lib.dora_norm_finalize.restype = c_i
        _lib = lib
        return lib


# ----------------------------------------------------------------- helpers

_DT = {torch.float32: DORA_F32, torch.bfloat16: DORA_BF16}


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype not in _DT:
        raise TypeError(f"unsupported dtype {t.dtype}: the library takes float32 or bfloat16")
    return _DT[t.dtype]


def _dev(t: Optional[torch.Tensor], name: str, dtype=None, shape=None) -> int:
    if t is None:
        return 0
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor (got {t.device})")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype} (got {t.dtype})")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)} (got {tuple(t.shape)})")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(status: int, where: str):
    if status != DORA_OK:
        raise DoraError(status, where)


def _workspace(nbytes: int, device, ws: Optional[torch.Tensor]) -> torch.Tensor:
    if ws is not None:
        return ws
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


# ----------------------------------------------------------------- API

def status_string(status: int) -> str:
    return load_library().dora_status_string(int(status)).decode()


def dora_version() -> int:
    return load_library().dora_version()


def dora_launch_count() -> int:
    return int(load_library().dora_launch_count())


def dora_set_wait_timeout_ns(ns: int) -> None:
    load_library().dora_set_wait_timeout_ns(int(ns))


def dora_set_timing_events(before: Optional[torch.cuda.Event], after: Optional[torch.cuda.Event]):
    """The next call on this thread records the two events around its
    principal kernel (see include/dora.h)."""
    load_library().dora_set_timing_events(before.cuda_event if before is not None else None,
                                          after.cuda_event if after is not None else None)


def dora_set_trace_buffer(buf: Optional[torch.Tensor]) -> None:
    """Diagnostics: per-CTA trace of the fused norm GEMM (see include/dora.h)."""
    load_library().dora_set_trace_buffer(_dev(buf, "trace", torch.int64) if buf is not None else None)


def dora_norm_plan_check(shapes: Sequence[Sequence[int]], grouped: bool = False,
                         pairs: int = 74) -> None:
    """Host-only self-check of the fused norm's schedule for modules of
    `shapes` [(d_out, d_in, r), ...] on `pairs` CTA pairs (see include/dora.h);
    raises DoraError naming the first invariant that fails."""
    n = len(shapes)
    arr = [(ctypes.c_int64 * n)(*[int(x[k]) for x in shapes]) for k in range(3)]
    _check(load_library().dora_norm_plan_check(arr[0], arr[1], arr[2], n, int(bool(grouped)),
                                               int(pairs)), "dora_norm_plan_check")


def dora_debug_unsignalled_wait(timeout_ns: int, stream=None) -> None:
    _check(load_library().dora_debug_unsignalled_wait(int(timeout_ns), _stream(stream)),
           "dora_debug_unsignalled_wait")


def dora_get_device_status(stream=None) -> int:
    return int(load_library().dora_get_device_status(_stream(stream)))


def dora_factored_norm_workspace_size(d_out: int, d_in: int, r: int, dtype: torch.dtype) -> int:
    return int(load_library().dora_factored_norm_workspace_size(d_out, d_in, r, _DT[dtype]))


def dora_factored_norm(W0: torch.Tensor, A: torch.Tensor, B: torch.Tensor, s: float,
                       m: Optional[torch.Tensor] = None, eps: float = 0.0,
                       n_out: Optional[torch.Tensor] = None, g_out: Optional[torch.Tensor] = None,
                       ws: Optional[torch.Tensor] = None, stream=None):
    """n = factored row norm of W0 + s B A (and g = m / max(n, eps) if m is given).
    Returns (n, g) with g None when m is None."""
    lib = load_library()
    dt = _dtype_code(W0)
    d_out, d_in = W0.shape
    r = A.shape[0]
    _dev(W0, "W0", W0.dtype)
    _dev(A, "A", W0.dtype, (r, d_in))
    _dev(B, "B", W0.dtype, (d_out, r))
    dev = W0.device
    if n_out is None:
        n_out = torch.empty(d_out, dtype=torch.float32, device=dev)
    if m is not None and g_out is None:
        g_out = torch.empty(d_out, dtype=torch.float32, device=dev)
    need = lib.dora_factored_norm_workspace_size(d_out, d_in, r, dt)
    ws = _workspace(need, dev, ws)
    _check(lib.dora_factored_norm(
        _dev(W0, "W0"), _dev(A, "A"), _dev(B, "B"), dt, d_out, d_in, r, float(s),
        _dev(m, "m", torch.float32, (d_out,)), float(eps),
        _dev(n_out, "n_out", torch.float32, (d_out,)),
        _dev(g_out, "g_out", torch.float32, (d_out,)),
        _dev(ws, "ws"), ws.numel() * ws.element_size(), _stream(stream)), "dora_factored_norm")
    return n_out, (g_out if m is not None else None)


def _problems(items: Sequence[dict]):
    arr = (NormProblem * len(items))()
    for i, p in enumerate(items):
        W0, A, B = p["W0"], p["A"], p["B"]
        d_out, d_in = W0.shape
        r = A.shape[0]
        arr[i].W0 = _dev(W0, f"W0[{i}]", torch.bfloat16)
        arr[i].A = _dev(A, f"A[{i}]", torch.bfloat16, (r, d_in))
        arr[i].B = _dev(B, f"B[{i}]", torch.bfloat16, (d_out, r))
        arr[i].m = _dev(p.get("m"), f"m[{i}]", torch.float32, (d_out,))
        arr[i].n_out = _dev(p["n_out"], f"n_out[{i}]", torch.float32, (d_out,))
        arr[i].g_out = _dev(p.get("g_out"), f"g_out[{i}]", torch.float32, (d_out,))
        arr[i].d_out, arr[i].d_in, arr[i].r = d_out, d_in, r
        arr[i].s = float(p["s"])
    return arr


def dora_factored_norm_grouped_workspace_size(items: Sequence[dict]) -> int:
    arr = _problems(items)
    return int(load_library().dora_factored_norm_grouped_workspace_size(arr, len(items), DORA_BF16))


def dora_factored_norm_grouped(items: Sequence[dict], eps: float = 0.0,
                               ws: Optional[torch.Tensor] = None, stream=None):
    """Grouped norm over modules given as dicts with keys W0, A, B, s, n_out and
    optionally m, g_out (bf16 weights, fp32 vectors)."""
    lib = load_library()
    arr = _problems(items)
    need = lib.dora_factored_norm_grouped_workspace_size(arr, len(items), DORA_BF16)
    ws = _workspace(need, items[0]["W0"].device, ws)
    _check(lib.dora_factored_norm_grouped(arr, len(items), DORA_BF16, float(eps), _dev(ws, "ws"),
                                          ws.numel() * ws.element_size(), _stream(stream)),
           "dora_factored_norm_grouped")


def dora_compose_fwd(base: torch.Tensor, lora: torch.Tensor, m: torch.Tensor, n: torch.Tensor,
                     s: float, eps: float = 0.0, y: Optional[torch.Tensor] = None, stream=None):
    """y = base + (g - 1) base + g s lora with g = m / max(n, eps)."""
    lib = load_library()
    dt = _dtype_code(base)
    T, d_out = base.shape
    if y is None:
        y = torch.empty_like(base)
    _check(lib.dora_compose_fwd(
        _dev(base, "base", base.dtype), _dev(lora, "lora", base.dtype, (T, d_out)),
        _dev(m, "m", torch.float32, (d_out,)), _dev(n, "n", torch.float32, (d_out,)), float(s),
        float(eps), dt, T, d_out, _dev(y, "y", base.dtype, (T, d_out)), _stream(stream)),
        "dora_compose_fwd")
    return y


def dora_compose_fwd_delta(base: torch.Tensor, lora: torch.Tensor, m: torch.Tensor,
                           n: torch.Tensor, s: float, eps: float = 0.0,
                           dy_out: Optional[torch.Tensor] = None, stream=None):
    """dY = (g - 1) base + g s lora with g = m / max(n, eps) (the caller adds Y_base)."""
    lib = load_library()
    dt = _dtype_code(base)
    T, d_out = base.shape
    if dy_out is None:
        dy_out = torch.empty_like(base)
    _check(lib.dora_compose_fwd_delta(
        _dev(base, "base", base.dtype), _dev(lora, "lora", base.dtype, (T, d_out)),
        _dev(m, "m", torch.float32, (d_out,)), _dev(n, "n", torch.float32, (d_out,)), float(s),
        float(eps), dt, T, d_out, _dev(dy_out, "dy_out", base.dtype, (T, d_out)),
        _stream(stream)),
        "dora_compose_fwd_delta")
    return dy_out


def dora_compose_bwd_workspace_size(T: int, d_out: int, dtype: torch.dtype) -> int:
    return int(load_library().dora_compose_bwd_workspace_size(T, d_out, _DT[dtype]))


def dora_compose_bwd(dy: torch.Tensor, base: torch.Tensor, lora: torch.Tensor, m: torch.Tensor,
                     n: torch.Tensor, s: float, eps: float = 0.0,
                     d_base: Optional[torch.Tensor] = None, d_lora: Optional[torch.Tensor] = None,
                     dm: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                     stream=None):
    """Returns (d_base, d_lora, dm)."""
    lib = load_library()
    dt = _dtype_code(dy)
    T, d_out = dy.shape
    dev = dy.device
    d_base = torch.empty_like(dy) if d_base is None else d_base
    d_lora = torch.empty_like(dy) if d_lora is None else d_lora
    dm = torch.empty(d_out, dtype=torch.float32, device=dev) if dm is None else dm
    need = lib.dora_compose_bwd_workspace_size(T, d_out, dt)
    ws = _workspace(need, dev, ws)
    _check(lib.dora_compose_bwd(
        _dev(dy, "dy", dy.dtype), _dev(base, "base", dy.dtype, (T, d_out)),
        _dev(lora, "lora", dy.dtype, (T, d_out)), _dev(m, "m", torch.float32, (d_out,)),
        _dev(n, "n", torch.float32, (d_out,)), float(s), float(eps), dt, T, d_out,
        _dev(d_base, "d_base", dy.dtype, (T, d_out)), _dev(d_lora, "d_lora", dy.dtype, (T, d_out)),
        _dev(dm, "dm", torch.float32, (d_out,)), _dev(ws, "ws"), ws.numel() * ws.element_size(),
        _stream(stream)), "dora_compose_bwd")
    return d_base, d_lora, dm


def dora_compose_bwd_static(dy: torch.Tensor, base: torch.Tensor, lora: torch.Tensor,
                            m: torch.Tensor, n: torch.Tensor, s: float, eps: float = 0.0,
                            d_base: Optional[torch.Tensor] = None,
                            d_lora: Optional[torch.Tensor] = None,
                            dm: Optional[torch.Tensor] = None, stream=None):
    """dora_compose_bwd without a workspace (the library's fixed scratch array;
    see include/dora.h for its size limit and sharing rules).  Returns
    (d_base, d_lora, dm)."""
    lib = load_library()
    dt = _dtype_code(dy)
    T, d_out = dy.shape
    dev = dy.device
    d_base = torch.empty_like(dy) if d_base is None else d_base
    d_lora = torch.empty_like(dy) if d_lora is None else d_lora
    dm = torch.empty(d_out, dtype=torch.float32, device=dev) if dm is None else dm
    _check(lib.dora_compose_bwd_static(
        _dev(dy, "dy", dy.dtype), _dev(base, "base", dy.dtype, (T, d_out)),
        _dev(lora, "lora", dy.dtype, (T, d_out)), _dev(m, "m", torch.float32, (d_out,)),
        _dev(n, "n", torch.float32, (d_out,)), float(s), float(eps), dt, T, d_out,
        _dev(d_base, "d_base", dy.dtype, (T, d_out)), _dev(d_lora, "d_lora", dy.dtype, (T, d_out)),
        _dev(dm, "dm", torch.float32, (d_out,)), _stream(stream)), "dora_compose_bwd_static")
    return d_base, d_lora, dm


def dora_compose_fwd_train(base: torch.Tensor, lora: torch.Tensor, m: torch.Tensor,
                           n: torch.Tensor, s: float, eps: float = 0.0,
                           y: Optional[torch.Tensor] = None, inner: Optional[torch.Tensor] = None,
                           stream=None):
    """Training forward: returns (y, inner) with inner = base + s lora."""
    lib = load_library()
    dt = _dtype_code(base)
    T, d_out = base.shape
    y = torch.empty_like(base) if y is None else y
    inner = torch.empty_like(base) if inner is None else inner
    _check(lib.dora_compose_fwd_train(
        _dev(base, "base", base.dtype), _dev(lora, "lora", base.dtype, (T, d_out)),
        _dev(m, "m", torch.float32, (d_out,)), _dev(n, "n", torch.float32, (d_out,)), float(s),
        float(eps), dt, T, d_out, _dev(y, "y", base.dtype, (T, d_out)),
        _dev(inner, "inner", base.dtype, (T, d_out)), _stream(stream)), "dora_compose_fwd_train")
    return y, inner


def dora_compose_bwd_inner(dy: torch.Tensor, inner: torch.Tensor, m: torch.Tensor,
                           n: torch.Tensor, s: float, eps: float = 0.0,
                           d_base: Optional[torch.Tensor] = None,
                           d_lora: Optional[torch.Tensor] = None,
                           dm: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                           stream=None):
    """Backward from inner = base + s lora.  Returns (d_base, d_lora, dm)."""
    lib = load_library()
    dt = _dtype_code(dy)
    T, d_out = dy.shape
    dev = dy.device
    d_base = torch.empty_like(dy) if d_base is None else d_base
    d_lora = torch.empty_like(dy) if d_lora is None else d_lora
    dm = torch.empty(d_out, dtype=torch.float32, device=dev) if dm is None else dm
    ws = _workspace(lib.dora_compose_bwd_workspace_size(T, d_out, dt), dev, ws)
    _check(lib.dora_compose_bwd_inner(
        _dev(dy, "dy", dy.dtype), _dev(inner, "inner", dy.dtype, (T, d_out)),
        _dev(m, "m", torch.float32, (d_out,)), _dev(n, "n", torch.float32, (d_out,)), float(s),
        float(eps), dt, T, d_out, _dev(d_base, "d_base", dy.dtype, (T, d_out)),
        _dev(d_lora, "d_lora", dy.dtype, (T, d_out)), _dev(dm, "dm", torch.float32, (d_out,)),
        _dev(ws, "ws"), ws.numel() * ws.element_size(), _stream(stream)),
        "dora_compose_bwd_inner")
    return d_base, d_lora, dm


def dora_compose_bwd_frozen(dy: torch.Tensor, m: torch.Tensor, n: torch.Tensor, s: float,
                            eps: float = 0.0, d_base: Optional[torch.Tensor] = None,
                            d_lora: Optional[torch.Tensor] = None, stream=None):
    """Backward with the magnitude frozen.  Returns (d_base, d_lora)."""
    lib = load_library()
    dt = _dtype_code(dy)
    T, d_out = dy.shape
    d_base = torch.empty_like(dy) if d_base is None else d_base
    d_lora = torch.empty_like(dy) if d_lora is None else d_lora
    _check(lib.dora_compose_bwd_frozen(
        _dev(dy, "dy", dy.dtype), _dev(m, "m", torch.float32, (d_out,)),
        _dev(n, "n", torch.float32, (d_out,)), float(s), float(eps), dt, T, d_out,
        _dev(d_base, "d_base", dy.dtype, (T, d_out)), _dev(d_lora, "d_lora", dy.dtype, (T, d_out)),
        _stream(stream)), "dora_compose_bwd_frozen")
    return d_base, d_lora


_COMPOSE_ACT = ("base", "lora", "inner", "y", "dy", "d_base", "d_lora")


def _compose_problems(items: Sequence[dict]):
    """ComposeProblem array from dicts: any of base, lora, inner, y, dy,
    d_base, d_lora ([T, d_out], one dtype), m, n, dm ([d_out] fp32), s."""
    arr = (ComposeProblem * len(items))()
    dtype = None
    for i, p in enumerate(items):
        ref = next(p[k] for k in _COMPOSE_ACT if p.get(k) is not None)
        T, d_out = ref.shape
        dtype = dtype or ref.dtype
        for k in _COMPOSE_ACT:
            setattr(arr[i], k, _dev(p.get(k), f"{k}[{i}]", dtype, (T, d_out)))
        arr[i].m = _dev(p["m"], f"m[{i}]", torch.float32, (d_out,))
        arr[i].n = _dev(p["n"], f"n[{i}]", torch.float32, (d_out,))
        arr[i].dm = _dev(p.get("dm"), f"dm[{i}]", torch.float32, (d_out,))
        arr[i].T, arr[i].d_out = T, d_out
        arr[i].s = float(p["s"])
    if dtype not in _DT:
        raise TypeError(f"unsupported dtype {dtype}: the library takes float32 or bfloat16")
    return arr, _DT[dtype]


def dora_compose_fwd_grouped(items: Sequence[dict], eps: float = 0.0, stream=None) -> None:
    """One launch over several modules (dicts with base, lora, m, n, s, y and
    optionally inner), written in place."""
    arr, dt = _compose_problems(items)
    _check(load_library().dora_compose_fwd_grouped(arr, len(items), dt, float(eps),
                                                   _stream(stream)), "dora_compose_fwd_grouped")


def dora_compose_bwd_grouped_workspace_size(items: Sequence[dict]) -> int:
    arr, dt = _compose_problems(items)
    return int(load_library().dora_compose_bwd_grouped_workspace_size(arr, len(items), dt))


def dora_compose_bwd_grouped(items: Sequence[dict], eps: float = 0.0,
                             ws: Optional[torch.Tensor] = None, stream=None) -> None:
    """Backward of several modules (dicts with dy, m, n, s, d_base, d_lora and
    dm plus inner, or base and lora; no dm: frozen magnitude), in place."""
    lib = load_library()
    arr, dt = _compose_problems(items)
    need = lib.dora_compose_bwd_grouped_workspace_size(arr, len(items), dt)
    dev = next(p[k] for k in _COMPOSE_ACT for p in items if p.get(k) is not None).device
    ws = _workspace(need, dev, ws) if need > 0 else None
    _check(lib.dora_compose_bwd_grouped(arr, len(items), dt, float(eps), _dev(ws, "ws"),
                                        0 if ws is None else ws.numel() * ws.element_size(),
                                        _stream(stream)), "dora_compose_bwd_grouped")


def dora_merge_weight_workspace_size(d_out: int, d_in: int, r: int) -> int:
    return int(load_library().dora_merge_weight_workspace_size(d_out, d_in, r))


def dora_merge_weight(W0: torch.Tensor, A: torch.Tensor, B: torch.Tensor, m: torch.Tensor,
                      n: torch.Tensor, s: float, eps: float = 0.0,
                      W_out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                      stream=None) -> torch.Tensor:
    """W' = g (W0 + s B A), g = m / max(n, eps), bf16 [d_out, d_in].  W_out may
    be W0 itself (in-place merge)."""
    lib = load_library()
    d_out, d_in = W0.shape
    r = A.shape[0]
    W_out = torch.empty_like(W0) if W_out is None else W_out
    ws = _workspace(lib.dora_merge_weight_workspace_size(d_out, d_in, r), W0.device, ws)
    _check(lib.dora_merge_weight(
        _dev(W0, "W0", torch.bfloat16), _dev(A, "A", torch.bfloat16, (r, d_in)),
        _dev(B, "B", torch.bfloat16, (d_out, r)), _dev(m, "m", torch.float32, (d_out,)),
        _dev(n, "n", torch.float32, (d_out,)), float(s), float(eps), d_out, d_in, r,
        _dev(W_out, "W_out", torch.bfloat16, (d_out, d_in)), _dev(ws, "ws"),
        ws.numel() * ws.element_size(), _stream(stream)), "dora_merge_weight")
    return W_out


def dora_factored_norm_sq(W0: torch.Tensor, A: torch.Tensor, B: torch.Tensor, s: float,
                          sq_out: Optional[torch.Tensor] = None,
                          ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Squared row-norm contribution of one column shard (W0[:, J], A[:, J],
    whole B), fp32 [d_out], before any clamp or square root."""
    lib = load_library()
    dt = _dtype_code(W0)
    d_out, d_in = W0.shape
    r = A.shape[0]
    dev = W0.device
    sq_out = torch.empty(d_out, dtype=torch.float32, device=dev) if sq_out is None else sq_out
    ws = _workspace(lib.dora_factored_norm_workspace_size(d_out, d_in, r, dt), dev, ws)
    _check(lib.dora_factored_norm_sq(
        _dev(W0, "W0", W0.dtype), _dev(A, "A", W0.dtype, (r, d_in)),
        _dev(B, "B", W0.dtype, (d_out, r)), dt, d_out, d_in, r, float(s),
        _dev(sq_out, "sq_out", torch.float32, (d_out,)), _dev(ws, "ws"),
        ws.numel() * ws.element_size(), _stream(stream)), "dora_factored_norm_sq")
    return sq_out


def dora_norm_finalize(sq: torch.Tensor, m: Optional[torch.Tensor] = None, eps: float = 0.0,
                       n_out: Optional[torch.Tensor] = None,
                       g_out: Optional[torch.Tensor] = None, stream=None):
    """n = sqrt(max(sq, 0)) and, with m, g = m / max(n, eps).  Returns (n, g or None)."""
    lib = load_library()
    d_out = sq.shape[0]
    dev = sq.device
    n_out = torch.empty(d_out, dtype=torch.float32, device=dev) if n_out is None else n_out
    if m is not None and g_out is None:
        g_out = torch.empty(d_out, dtype=torch.float32, device=dev)
    _check(lib.dora_norm_finalize(
        _dev(sq, "sq", torch.float32, (d_out,)), _dev(m, "m", torch.float32, (d_out,)),
        float(eps), d_out, _dev(n_out, "n_out", torch.float32, (d_out,)),
        _dev(g_out if m is not None else None, "g_out", torch.float32, (d_out,)),
        _stream(stream)), "dora_norm_finalize")
    return n_out, (g_out if m is not None else None)
