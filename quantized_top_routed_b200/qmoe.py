"""ctypes binding of libqmoe.so (C ABI in include/qmoe.h).

Every function here marshals arguments and calls the C entry point of the
same name; all of the layer's computation happens in the library's CUDA
kernels.  Pointer arguments accept an int (device address), ``None``
(NULL) or any object with ``data_ptr()`` (a torch tensor).  A non-zero
status raises :class:`QmoeError` with the library's message.

There is no fallback: if the library cannot be built or loaded the import
of the handle functions fails.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

from . import build as _build

QMOE_OK = 0
QMOE_ERR_INVALID = 1
QMOE_ERR_UNSUPPORTED = 2
QMOE_ERR_CUDA = 3
QMOE_ERR_OOM = 4
QMOE_ERR_TIMEOUT = 5
QMOE_ERR_BOUNDS = 6

W_INT8_PC = 1
W_INT4_G128 = 2
W_FP8_E4M3_PC = 3

STAGES = ("router", "schedule", "gate_up", "down", "combine")

EXPORTS = ("qmoe_create", "qmoe_route", "qmoe_forward", "qmoe_forward_host", "qmoe_check_error",
           "qmoe_profile", "qmoe_profile_read", "qmoe_launches_per_forward", "qmoe_destroy",
           "qmoe_last_error", "qmoe_route_topk_noalloc", "qmoe_set_wait_limit", "qmoe_debug_build")


class QmoeError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"qmoe status {status}: {message}")
        self.status = status


class qmoe_config(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("E", ctypes.c_int32), ("k", ctypes.c_int32),
                ("I", ctypes.c_int32), ("n_shared", ctypes.c_int32), ("max_tokens", ctypes.c_int32)]


class qmoe_expert(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("w13", ctypes.c_void_p), ("s13", ctypes.c_void_p),
                ("w2", ctypes.c_void_p), ("s2", ctypes.c_void_p)]


_lib = None


def debug_requested() -> bool:
    """QMOE_DEBUG=1 in the environment selects the bounds-checking build."""
    return os.environ.get("QMOE_DEBUG") == "1"


def library_path() -> str:
    return _build.LIB_DEBUG if debug_requested() else _build.LIB


def load(build_if_missing: bool = True) -> ctypes.CDLL:
    """Load libqmoe.so, or libqmoe_debug.so when QMOE_DEBUG=1 (building it
    in-tree first when it is missing or stale)."""
    global _lib
    if _lib is not None:
        return _lib
    debug = debug_requested()
    path = library_path()
    if build_if_missing and not (_build.up_to_date(debug=True) if debug else _build.up_to_date()):
        _build.build(debug=debug)
    if not os.path.exists(path):
        raise OSError(f"{path} is missing; run python -m quantized_top_routed_b200.build")
    lib = ctypes.CDLL(path)
    vp, i32, f32p = ctypes.c_void_p, ctypes.c_int32, ctypes.POINTER(ctypes.c_float)
    lib.qmoe_create.argtypes = [ctypes.POINTER(qmoe_config), vp, vp, ctypes.POINTER(qmoe_expert),
                                ctypes.POINTER(vp)]
    lib.qmoe_route.argtypes = [vp, vp, vp, i32, vp, vp, vp, vp, vp, vp, vp]
    lib.qmoe_forward.argtypes = [vp, vp, i32, vp, vp]
    lib.qmoe_forward_host.argtypes = [vp, vp, i32, vp, vp]
    lib.qmoe_check_error.argtypes = [vp, vp]
    lib.qmoe_profile.argtypes = [vp, i32]
    lib.qmoe_profile_read.argtypes = [vp, f32p, i32, ctypes.POINTER(i32)]
    lib.qmoe_launches_per_forward.argtypes = [vp, i32]
    lib.qmoe_launches_per_forward.restype = i32
    lib.qmoe_destroy.argtypes = [vp]
    lib.qmoe_last_error.argtypes = []
    lib.qmoe_last_error.restype = ctypes.c_char_p
    lib.qmoe_route_topk_noalloc.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, vp, vp]
    lib.qmoe_set_wait_limit.argtypes = [vp, ctypes.c_int64]
    lib.qmoe_debug_build.argtypes = []
    lib.qmoe_debug_build.restype = i32
    for name in ("qmoe_create", "qmoe_route", "qmoe_forward", "qmoe_forward_host", "qmoe_check_error",
                 "qmoe_profile", "qmoe_profile_read", "qmoe_destroy", "qmoe_route_topk_noalloc",
                 "qmoe_set_wait_limit"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return int(x.data_ptr())
    if isinstance(x, ctypes.c_void_p):
        return x.value
    raise TypeError(f"cannot pass {type(x)} as a pointer")


def _stream(s) -> Optional[int]:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return int(s.cuda_stream)


def _check(status: int):
    if status != QMOE_OK:
        raise QmoeError(status, load().qmoe_last_error().decode())


def qmoe_last_error() -> str:
    return load().qmoe_last_error().decode()


def qmoe_create(d: int, E: int, k: int, I: int, n_shared: int, max_tokens: int, router_w, router_bias,
                experts: Sequence[tuple]) -> int:
    """experts: one (fmt, w13, s13, w2, s2) tuple per routed then shared expert."""
    lib = load()
    cfg = qmoe_config(d, E, k, I, n_shared, max_tokens)
    arr = (qmoe_expert * len(experts))()
    for i, (fmt, w13, s13, w2, s2) in enumerate(experts):
        arr[i] = qmoe_expert(fmt, _ptr(w13), _ptr(s13), _ptr(w2), _ptr(s2))
    h = ctypes.c_void_p()
    _check(lib.qmoe_create(ctypes.byref(cfg), _ptr(router_w), _ptr(router_bias), arr, ctypes.byref(h)))
    return h.value


def qmoe_route(h: int, x, logits, T: int, topk_idx, topk_gate, counts, offsets, sorted_token, inv_pos,
               stream=None):
    _check(load().qmoe_route(h, _ptr(x), _ptr(logits), T, _ptr(topk_idx), _ptr(topk_gate), _ptr(counts),
                             _ptr(offsets), _ptr(sorted_token), _ptr(inv_pos), _stream(stream)))


def qmoe_forward(h: int, x, T: int, out, stream=None):
    _check(load().qmoe_forward(h, _ptr(x), T, _ptr(out), _stream(stream)))


def qmoe_forward_host(h: int, x_host, T: int, out_host, stream=None):
    _check(load().qmoe_forward_host(h, _ptr(x_host), T, _ptr(out_host), _stream(stream)))


def qmoe_check_error(h: int, stream=None):
    _check(load().qmoe_check_error(h, _stream(stream)))


def qmoe_set_wait_limit(h: int, cycles: int):
    """Bound (SM cycles) of the grouped GEMMs' barrier waits; 0 = default."""
    _check(load().qmoe_set_wait_limit(h, cycles))


def qmoe_profile(h: int, enable: bool):
    _check(load().qmoe_profile(h, 1 if enable else 0))


def qmoe_profile_read(h: int):
    """Returns ({stage: total ms}, number of forwards recorded)."""
    ms = (ctypes.c_float * len(STAGES))()
    calls = ctypes.c_int32()
    _check(load().qmoe_profile_read(h, ms, len(STAGES), ctypes.byref(calls)))
    return {name: float(ms[i]) for i, name in enumerate(STAGES)}, int(calls.value)


def qmoe_launches_per_forward(h: int, T: int) -> int:
    return int(load().qmoe_launches_per_forward(h, T))


def qmoe_destroy(h: Optional[int]):
    _check(load().qmoe_destroy(h))


# Sizes the no-allocation router accepts (T * E logits at most).
QMOE_ROUTE_STATIC_MAX_LOGITS = 1 << 20


def qmoe_route_topk_noalloc(x, router_w, router_bias, T: int, d: int, E: int, k: int, topk_idx, topk_gate,
                            stream=None):
    """Router stage without a handle, using the library's fixed scratch
    array instead of allocating (for callers that cannot allocate device
    memory mid-step).  Calls that may overlap on one GPU race."""
    _check(load().qmoe_route_topk_noalloc(_ptr(x), _ptr(router_w), _ptr(router_bias), T, d, E, k,
                                          _ptr(topk_idx), _ptr(topk_gate), _stream(stream)))


# ---------------------------------------------------------------------------
# convenience: put a generated layer on the device and create its handle
# ---------------------------------------------------------------------------
class DeviceLayer:
    """Device copies of a ``synth.LayerInputs`` and a qmoe handle built from them.

    The canonical weight buffers are freed once the handle holds its own
    re-laid-out copy.
    """

    def __init__(self, layer, max_tokens: Optional[int] = None, device: str = "cuda"):
        import numpy as np
        import torch

        def dev(a):
            a = np.ascontiguousarray(a)
            if a.dtype == np.uint16:          # bf16 bit patterns
                a = a.view(np.int16)
            return torch.from_numpy(a).to(device)

        self.layer = layer
        self.max_tokens = max_tokens or layer.T
        router_w = dev(layer.router_w)
        router_b = dev(layer.router_b) if layer.router_b is not None else None
        experts, keep = [], []
        for ex in layer.experts:
            t = (dev(ex.w13.view(np.uint8)), dev(ex.s13), dev(ex.w2.view(np.uint8)), dev(ex.s2))
            keep.append(t)
            experts.append((ex.fmt, *t))
        self.handle = qmoe_create(layer.d, layer.E, layer.k, layer.I, layer.S, self.max_tokens, router_w,
                                  router_b, experts)
        del keep, experts, router_w, router_b
        self.x = dev(layer.x.view(np.int16))

    def close(self):
        if self.handle:
            qmoe_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
