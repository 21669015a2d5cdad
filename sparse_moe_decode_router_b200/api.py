"""Python binding of libmoe_decode.so (include/moe_decode.h).

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels.  Functions carry the C names; tensors may be passed as torch
tensors (their data_ptr is used) or as integer addresses.  A non-OK status
raises MoEError.  There is no fallback: without the built library (or
without a GPU) calls fail.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_decode.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_CUDA = 3
MOE_ERR_OOM = 4
MOE_ERR_TIMEOUT = 5

MOE_FLAG_NO_PDL = 0x1
MOE_FLAG_SIDE_STREAM = 0x2
MOE_FLAG_NO_PREFETCH = 0x4
MOE_FLAG_NO_GROUPED = 0x8
MOE_FLAG_MX_EXPERTS = 0x10
MOE_FLAG_WARP_MMA = 0x80
MOE_PATH_GEMV, MOE_PATH_GROUPED, MOE_PATH_TCGEN05 = 0, 1, 2
MOE_FLAG_ROUTER_SIGMOID = 0x20
MOE_FLAG_PERSISTENT = 0x40

# every entry point the header declares
EXPORTS = (
    "moe_layer_create", "moe_layer_destroy", "moe_router_topk", "moe_experts_mxfp4",
    "moe_combine_residual", "moe_layer_forward", "moe_layer_forward_host", "moe_layer_routing",
    "moe_layer_last_device_error", "moe_layer_set_probe", "moe_router_topk_noalloc",
    "moe_router_topk_noalloc_last_error", "moe_selftest", "moe_layer_expert_path",
    "moe_status_string",
)

MOE_SELFTEST_WAIT_TIMEOUT = 1
MOE_SELFTEST_FAIL_NEXT_ALLOC = 2


class MoEError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {moe_status_string(status)} ({status})")


class moe_layer_config(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("n_experts", ctypes.c_int), ("top_k", ctypes.c_int),
                ("inter", ctypes.c_int), ("shared_inter", ctypes.c_int), ("max_batch", ctypes.c_int),
                ("flags", ctypes.c_uint)]


class moe_layer_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "router_w", "router_bias", "w_gate_up", "s_gate_up", "w_down", "s_down",
        "shared_gate_up", "shared_down", "shared_mx_gate_up", "shared_mx_s_gate_up",
        "shared_mx_down", "shared_mx_s_down")]


class moe_routing(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "topk_idx", "topk_w", "counts", "offsets", "pair_ids", "active", "n_active")]


_LIB = None


def load_library(path: str = LIB_PATH):
    """Load the shared library (raises if it is missing)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is not built; run __graft_entry__.build()")
    L = ctypes.CDLL(path)
    vp, i32, st = ctypes.c_void_p, ctypes.c_int, ctypes.c_int
    sig = {
        "moe_layer_create": [ctypes.POINTER(moe_layer_config), ctypes.POINTER(moe_layer_weights),
                             ctypes.POINTER(vp)],
        "moe_layer_destroy": [vp],
        "moe_router_topk": [vp, vp, i32, ctypes.POINTER(moe_routing), vp],
        "moe_experts_mxfp4": [vp, vp, i32, ctypes.POINTER(moe_routing), vp, vp, vp],
        "moe_combine_residual": [vp, i32, ctypes.POINTER(moe_routing), vp, vp, vp, vp, vp],
        "moe_layer_forward": [vp, vp, vp, vp, vp, i32, vp],
        "moe_layer_forward_host": [vp, vp, vp, vp, i32, vp],
        "moe_layer_routing": [vp, ctypes.POINTER(moe_routing)],
        "moe_layer_last_device_error": [vp],
        "moe_layer_set_probe": [vp, vp, vp],
        "moe_router_topk_noalloc": [vp, vp, i32, i32, i32, vp, i32, ctypes.POINTER(moe_routing), vp],
        "moe_router_topk_noalloc_last_error": [],
        "moe_selftest": [i32, vp],
    }
    for name, args in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = st
    L.moe_layer_expert_path.argtypes = [vp, i32]
    L.moe_layer_expert_path.restype = ctypes.c_int
    L.moe_status_string.argtypes = [ctypes.c_int]
    L.moe_status_string.restype = ctypes.c_char_p
    _LIB = L
    return L


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(s) -> int | None:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream if hasattr(s, "cuda_stream") else int(s)


def _check(fn: str, rc: int):
    if rc != MOE_OK:
        raise MoEError(fn, rc)


def moe_status_string(status: int) -> str:
    return load_library().moe_status_string(int(status)).decode()


def make_routing(topk_idx, topk_w, counts, offsets, pair_ids, active, n_active) -> moe_routing:
    return moe_routing(*(_ptr(t) for t in (topk_idx, topk_w, counts, offsets, pair_ids, active, n_active)))


def moe_layer_create(cfg: moe_layer_config, weights: moe_layer_weights) -> int:
    h = ctypes.c_void_p()
    _check("moe_layer_create", load_library().moe_layer_create(ctypes.byref(cfg), ctypes.byref(weights),
                                                                ctypes.byref(h)))
    return h.value


def moe_layer_destroy(layer: int):
    _check("moe_layer_destroy", load_library().moe_layer_destroy(layer))


def moe_router_topk(layer: int, x, B: int, routing: moe_routing | None = None, stream=None):
    _check("moe_router_topk", load_library().moe_router_topk(
        layer, _ptr(x), B, None if routing is None else ctypes.byref(routing), _stream(stream)))


def moe_experts_mxfp4(layer: int, x, B: int, routing, y_routed, y_shared, stream=None):
    _check("moe_experts_mxfp4", load_library().moe_experts_mxfp4(
        layer, _ptr(x), B, None if routing is None else ctypes.byref(routing), _ptr(y_routed),
        _ptr(y_shared), _stream(stream)))


def moe_combine_residual(layer: int, B: int, routing, y_routed, y_shared, residual, out, stream=None):
    _check("moe_combine_residual", load_library().moe_combine_residual(
        layer, B, None if routing is None else ctypes.byref(routing), _ptr(y_routed), _ptr(y_shared),
        _ptr(residual), _ptr(out), _stream(stream)))


def moe_layer_forward(layer: int, next_layer: int | None, x, residual, out, B: int, stream=None):
    _check("moe_layer_forward", load_library().moe_layer_forward(
        layer, next_layer, _ptr(x), _ptr(residual), _ptr(out), B, _stream(stream)))


def moe_layer_forward_host(layer: int, x_host, residual_host, out_host, B: int, stream=None):
    _check("moe_layer_forward_host", load_library().moe_layer_forward_host(
        layer, _ptr(x_host), _ptr(residual_host), _ptr(out_host), B, _stream(stream)))


def moe_layer_expert_path(layer: int, B: int) -> int:
    """MOE_PATH_* of the kernels a call at batch B runs the routed experts on."""
    p = load_library().moe_layer_expert_path(layer, B)
    if p < 0:
        raise ValueError(f"moe_layer_expert_path: bad layer or batch {B}")
    return p


def moe_layer_routing(layer: int) -> moe_routing:
    r = moe_routing()
    _check("moe_layer_routing", load_library().moe_layer_routing(layer, ctypes.byref(r)))
    return r


def moe_layer_last_device_error(layer: int) -> int:
    return int(load_library().moe_layer_last_device_error(layer))


def moe_layer_set_probe(layer: int, start_event=None, stop_event=None):
    s = None if start_event is None else start_event.cuda_event
    e = None if stop_event is None else stop_event.cuda_event
    _check("moe_layer_set_probe", load_library().moe_layer_set_probe(layer, s, e))


def moe_router_topk_noalloc(router_w_em, router_bias, hidden: int, n_experts: int, top_k: int, x, B: int,
                            routing: moe_routing, stream=None):
    """Router + top-k + bucketing with no device allocation (see the header).
    router_w_em is the expert-major [E][H] bf16 router matrix."""
    _check("moe_router_topk_noalloc", load_library().moe_router_topk_noalloc(
        _ptr(router_w_em), _ptr(router_bias), hidden, n_experts, top_k, _ptr(x), B, ctypes.byref(routing),
        _stream(stream)))


def moe_router_topk_noalloc_last_error() -> int:
    """Reads and clears the allocation-free router's device error word of the
    current device (see the header); returns the status code."""
    return int(load_library().moe_router_topk_noalloc_last_error())


def moe_selftest(what: int, stream=None) -> int:
    """Failure-path self-test (see the header); returns the status code."""
    return int(load_library().moe_selftest(int(what), _stream(stream)))
