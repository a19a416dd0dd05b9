"""The C-ABI library builds, loads and exports what include/qmoe.h declares (CPU only).

Only calls that fail argument validation before touching CUDA are made here.
"""
import ctypes
import os
import re

import pytest

from quantized_top_routed_b200 import qmoe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    with open(os.path.join(ROOT, "include", "qmoe.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qmoe_[a-z_]+)\s*\(", text)))


def test_library_loads_and_exports_every_declared_symbol():
    lib = qmoe.load()
    names = declared_functions()
    assert len(names) >= 8
    for name in names:
        assert hasattr(lib, name), f"{name} declared in qmoe.h but not exported"
    assert set(names) == set(qmoe.EXPORTS)


def test_symbols_are_c_linkage():
    out = os.popen(f"nm -D --defined-only {qmoe.library_path()}").read()
    for name in declared_functions():
        assert re.search(rf"\sT {name}$", out, flags=re.M), name


def test_destroy_null_is_ok_and_last_error_is_a_string():
    qmoe.qmoe_destroy(None)
    assert isinstance(qmoe.qmoe_last_error(), str)


def _create_raw(cfg, router_w=1, experts_n=1, fmt=1, ptrs=(16, 16, 16, 16)):
    lib = qmoe.load()
    arr = (qmoe.qmoe_expert * experts_n)()
    for i in range(experts_n):
        arr[i] = qmoe.qmoe_expert(fmt, *ptrs)
    h = ctypes.c_void_p(12345)
    st = lib.qmoe_create(ctypes.byref(cfg) if cfg is not None else None, router_w, arr, arr, ctypes.byref(h))
    return st, h.value


@pytest.mark.parametrize("cfg_kw,why", [
    (dict(d=100, E=8, k=2, I=512, n_shared=0, max_tokens=64), "d"),
    (dict(d=256, E=8, k=2, I=500, n_shared=0, max_tokens=64), "I"),
    (dict(d=256, E=0, k=1, I=512, n_shared=0, max_tokens=64), "E"),
    (dict(d=256, E=300, k=2, I=512, n_shared=0, max_tokens=64), "E"),
    (dict(d=256, E=8, k=9, I=512, n_shared=0, max_tokens=64), "k"),
    (dict(d=256, E=32, k=17, I=512, n_shared=0, max_tokens=64), "k"),
    (dict(d=256, E=8, k=2, I=512, n_shared=9, max_tokens=64), "n_shared"),
    (dict(d=256, E=8, k=2, I=512, n_shared=0, max_tokens=0), "max_tokens"),
])
def test_create_rejects_bad_shapes(cfg_kw, why):
    cfg = qmoe.qmoe_config(**cfg_kw)
    st, h = _create_raw(cfg, experts_n=max(1, cfg_kw["E"] + cfg_kw["n_shared"]))
    assert st == qmoe.QMOE_ERR_INVALID
    assert h is None
    assert why in qmoe.qmoe_last_error()


def test_create_rejects_null_and_unknown_format():
    st, _ = _create_raw(None)
    assert st == qmoe.QMOE_ERR_INVALID
    cfg = qmoe.qmoe_config(256, 2, 1, 256, 0, 4)
    st, _ = _create_raw(cfg, experts_n=2, fmt=7)
    assert st == qmoe.QMOE_ERR_INVALID and "format" in qmoe.qmoe_last_error()
    st, _ = _create_raw(cfg, experts_n=2, ptrs=(16, None, 16, 16))
    assert st == qmoe.QMOE_ERR_INVALID and "NULL" in qmoe.qmoe_last_error()


def test_calls_reject_null_handle():
    with pytest.raises(qmoe.QmoeError) as ei:
        qmoe.qmoe_forward(None, 16, 4, 16)
    assert ei.value.status == qmoe.QMOE_ERR_INVALID
    with pytest.raises(qmoe.QmoeError):
        qmoe.qmoe_route(None, 16, None, 4, 16, 16, 16, 16, 16, 16)
    with pytest.raises(qmoe.QmoeError):
        qmoe.qmoe_check_error(None)
    with pytest.raises(qmoe.QmoeError) as ei:
        qmoe.qmoe_set_wait_limit(None, 1000)
    assert ei.value.status == qmoe.QMOE_ERR_INVALID


@pytest.mark.parametrize("T,d,E,k,why", [
    (0, 256, 8, 2, "T must be"),
    (4, 200, 8, 2, "multiple of 128"),
    (4, 256, 300, 2, "E must be"),
    (4, 256, 8, 9, "k must be"),
    (qmoe.QMOE_ROUTE_STATIC_MAX_LOGITS // 8 + 1, 256, 8, 2, "exceeds the fixed routing scratch"),
])
def test_noalloc_route_validates_before_touching_the_device(T, d, E, k, why):
    # fake (never dereferenced) pointers: validation rejects before any CUDA call
    with pytest.raises(qmoe.QmoeError) as ei:
        qmoe.qmoe_route_topk_noalloc(16, 16, None, T, d, E, k, 16, 16)
    assert ei.value.status == qmoe.QMOE_ERR_INVALID
    assert why in str(ei.value)


def test_the_product_library_is_not_the_debug_build():
    assert qmoe.load().qmoe_debug_build() == 0


def test_debug_library_builds_and_exports_the_same_symbols():
    """The QMOE_DEBUG twin (device-side bounds checks that raise
    QMOE_ERR_BOUNDS instead of faulting) builds from the same sources and has
    the same C ABI; it reports itself through qmoe_debug_build()."""
    path = qmoe._build.build(debug=True)
    assert path == qmoe._build.LIB_DEBUG and qmoe._build.up_to_date(debug=True)
    lib = ctypes.CDLL(path)
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} missing from the debug build"
    lib.qmoe_debug_build.restype = ctypes.c_int32
    assert lib.qmoe_debug_build() == 1
