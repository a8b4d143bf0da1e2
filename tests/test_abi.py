"""The C-ABI library loads and exports every symbol include/moeq.h declares,
and its host-side argument checks answer without touching a GPU."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moeq.h")


def declared_symbols():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"MOEQ_API\s+[\w\s\*]+?\b(moeq_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def moeq():
    from bit_quantized_moe_routed_b200 import build
    build.build()
    from bit_quantized_moe_routed_b200 import moeq as m
    return m


def test_header_declares_the_entry_points():
    syms = declared_symbols()
    for s in ("moeq_layer_create", "moeq_upload_weights", "moeq_forward", "moeq_dequant",
              "moeq_layer_destroy", "moeq_layer_status", "moeq_status_string", "moeq_route",
              "moeq_forward_host", "moeq_forward_profiled", "moeq_route_noalloc", "moeq_router_upload",
              "moeq_router", "moeq_forward_routed", "moeq_vq_encode", "moeq_kernel_launches"):
        assert s in syms


def test_library_exports_every_declared_symbol(moeq):
    lib = C.CDLL(moeq.LIB_PATH)
    for s in declared_symbols():
        assert hasattr(lib, s), s
    assert sorted(moeq.EXPORTS) == declared_symbols()


def test_status_strings(moeq):
    for code in range(8):
        assert moeq.status_string(code)
    assert moeq.status_string(0) == "ok"
    assert moeq.status_string(99) == "unknown status"


def _desc(moeq, **kw):
    d = dict(hidden=256, inter=128, n_experts=16, top_k=2, max_tokens=4, fmt=0, act=0, device=0)
    d.update(kw)
    return moeq.LayerDesc(**d)


@pytest.mark.parametrize("bad", [
    dict(hidden=0), dict(inter=-1), dict(n_experts=0), dict(top_k=0), dict(max_tokens=0),
    dict(top_k=17), dict(n_experts=2048, top_k=2), dict(top_k=65, n_experts=128),
    dict(hidden=250), dict(inter=100), dict(hidden=320), dict(inter=96), dict(hidden=1152), dict(fmt=1, hidden=288), dict(fmt=2, inter=96),
    dict(fmt=5), dict(fmt=3, hidden=288), dict(fmt=4, inter=96), dict(act=2),
])
def test_create_rejects_bad_descriptors_on_the_host(moeq, bad):
    lib = moeq.lib()
    d = _desc(moeq, **bad)
    h = C.c_void_p(1234)
    assert lib.moeq_layer_create(C.byref(d), C.byref(h)) == moeq.INVALID_ARGUMENT
    assert h.value is None


def test_null_handles_are_rejected(moeq):
    lib = moeq.lib()
    assert lib.moeq_layer_create(None, None) == moeq.INVALID_ARGUMENT
    assert lib.moeq_forward(None, None, None, None, 1, None, None) == moeq.INVALID_ARGUMENT
    assert lib.moeq_forward_host(None, None, None, None, 1, None, None) == moeq.INVALID_ARGUMENT
    assert lib.moeq_dequant(None, 0, 0, None, None) == moeq.INVALID_ARGUMENT
    assert lib.moeq_route(None, None, 1, None, None, None) == moeq.INVALID_ARGUMENT
    assert lib.moeq_layer_status(None, 0) == moeq.INVALID_ARGUMENT
    assert lib.moeq_upload_weights(None, None, None) == moeq.INVALID_ARGUMENT
    lib.moeq_layer_destroy(None)   # no-op
