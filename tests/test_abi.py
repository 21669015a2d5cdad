"""CPU checks of the C-ABI library: it loads, exports every entry point the
header declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_decode.h")


def declared_symbols():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", txt)))


@pytest.fixture(scope="module")
def lib():
    from sparse_moe_decode_router_b200 import api
    return api.load_library()


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ("moe_layer_create", "moe_router_topk", "moe_experts_mxfp4", "moe_combine_residual",
                 "moe_layer_forward"):
        assert name in syms


def test_library_exports_every_declared_symbol(lib):
    from sparse_moe_decode_router_b200 import api
    syms = declared_symbols()
    assert sorted(api.EXPORTS) == syms
    for name in syms:
        assert hasattr(lib, name), name


def test_status_strings(lib):
    from sparse_moe_decode_router_b200 import api
    assert api.moe_status_string(0) == "ok"
    assert "invalid" in api.moe_status_string(1)
    assert "timed out" in api.moe_status_string(5)


def test_host_side_argument_checks(lib):
    from sparse_moe_decode_router_b200 import api
    # null config / weights / handle: rejected before touching the device
    assert lib.moe_layer_create(None, None, None) == api.MOE_ERR_INVALID_ARG
    h = ctypes.c_void_p()
    cfg = api.moe_layer_config(256, 32, 4, 128, 128, 1, 0)
    assert lib.moe_layer_create(ctypes.byref(cfg), None, ctypes.byref(h)) == api.MOE_ERR_INVALID_ARG
    w = api.moe_layer_weights(*([0x1000] * 8))
    for bad in (api.moe_layer_config(250, 32, 4, 128, 128, 1, 0),    # H not a multiple of 32
                api.moe_layer_config(256, 32, 40, 128, 128, 1, 0),   # k > 32
                api.moe_layer_config(256, 32, 4, 128, 128, 65, 0),   # max_batch > 64
                api.moe_layer_config(256, 2000, 4, 128, 128, 1, 0)): # E > 1024
        assert lib.moe_layer_create(ctypes.byref(bad), ctypes.byref(w), ctypes.byref(h)) == api.MOE_ERR_INVALID_ARG
    misaligned = api.moe_layer_weights(0x1008, None, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000, 0x1000)
    assert lib.moe_layer_create(ctypes.byref(cfg), ctypes.byref(misaligned), ctypes.byref(h)) == api.MOE_ERR_INVALID_ARG
    assert lib.moe_router_topk(None, 0x1000, 1, None, None) == api.MOE_ERR_INVALID_ARG
    assert lib.moe_layer_forward(None, None, 0x1000, 0x1000, 0x1000, 1, None) == api.MOE_ERR_INVALID_ARG
    assert lib.moe_layer_destroy(None) == api.MOE_OK
    with pytest.raises(api.MoEError):
        api.moe_layer_forward(None, None, 0x1000, 0x1000, 0x1000, 1)


def test_selftest_rejects_unknown_requests():
    """Host-side argument check of the failure-path self-test (no CUDA call)."""
    from sparse_moe_decode_router_b200 import api
    api.load_library()
    assert api.moe_selftest(0) == api.MOE_ERR_INVALID_ARG
    assert api.moe_selftest(99) == api.MOE_ERR_INVALID_ARG


def test_noalloc_router_rejects_invalid_calls_on_the_host(lib):
    """Every call here is refused by the host-side checks before any CUDA
    call, so the placeholder addresses are never dereferenced."""
    from sparse_moe_decode_router_b200 import api
    routing = api.make_routing(*([0x1000] * 7))

    def call(w=0x1000, H=256, E=32, k=4, x=0x1000, B=1, r=routing):
        return lib.moe_router_topk_noalloc(w, None, H, E, k, x, B, None if r is None else ctypes.byref(r), None)

    bad = [dict(w=None), dict(w=0x1008), dict(x=None), dict(x=0x1004), dict(r=None),
           dict(r=api.make_routing(*([0x1000] * 6 + [None]))),
           dict(H=0), dict(H=250), dict(H=16384 + 32),
           dict(E=0), dict(E=1025), dict(E=31), dict(E=1023, k=4), dict(k=0), dict(k=33, E=64),
           dict(k=8, E=4), dict(B=0), dict(B=65)]
    for kw in bad:
        assert call(**kw) == api.MOE_ERR_INVALID_ARG, kw
