"""ORACLE -- test infrastructure only.

ctypes front end of moe_oracle.cpp, the plain fp64 CPU implementation of the
sparse MXFP4 MoE decode layer that the CUDA library is checked against.
Only tests/, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
bench.py may import this package; the library itself never does.

Pins (tests/test_oracle_pins.py) tie every function here to something other
than itself: a hand-written E2M1 x E8M0 table, brute-force top-k over all
subsets, closed forms for the routing weights, bucket invariants, dense FFNs
on exactly representable weights, and special cases of the whole layer.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB = None


def lib_path() -> str:
    return os.path.join(_HERE, "liboracle.so")


def build(verbose=False) -> str:
    src = os.path.join(_HERE, "moe_oracle.cpp")
    cmd = ["g++", "-O2", "-std=c++17", "-fopenmp", "-fPIC", "-shared", "-o", lib_path(), src]
    if verbose:
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    return lib_path()


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def lib():
    global _LIB
    if _LIB is None:
        src = os.path.join(_HERE, "moe_oracle.cpp")
        if not os.path.exists(lib_path()) or os.path.getmtime(lib_path()) < os.path.getmtime(src):
            build()
        L = ctypes.CDLL(lib_path())
        vp, i32, dbl = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        L.oracle_e2m1_value.argtypes = [i32]
        L.oracle_e2m1_value.restype = dbl
        L.oracle_e8m0_value.argtypes = [i32]
        L.oracle_e8m0_value.restype = dbl
        L.oracle_round_bf16.argtypes = [dbl]
        L.oracle_round_bf16.restype = ctypes.c_uint16
        L.oracle_silu.argtypes = [dbl]
        L.oracle_silu.restype = dbl
        L.oracle_dequant_row.argtypes = [vp, vp, i32, vp]
        L.oracle_router_logits.argtypes = [vp, vp, vp, i32, i32, i32, vp]
        L.oracle_topk_softmax.argtypes = [vp, i32, i32, i32, vp, vp]
        L.oracle_bucket.argtypes = [vp, i32, i32, i32, vp, vp, vp, vp, vp]
        L.oracle_expert_ffn.argtypes = [vp, vp, vp, vp, vp, i32, i32, vp, vp]
        L.oracle_shared_ffn.argtypes = [vp, vp, vp, i32, i32, vp, vp]
        L.oracle_layer.argtypes = [i32] * 6 + [vp] * 11 + [i32] + [vp] * 13
        L.oracle_layer.restype = i32
        L.oracle_layer_v.argtypes = [i32] * 6 + [vp] * 11 + [i32] + [vp] * 13 + [i32] + [vp] * 4
        L.oracle_layer_v.restype = i32
        L.oracle_topk_sigmoid.argtypes = [vp, vp, i32, i32, i32, vp, vp]
        _LIB = L
    return _LIB


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---- single steps ----------------------------------------------------------
def e2m1_value(code: int) -> float:
    return lib().oracle_e2m1_value(int(code))


def e8m0_value(s: int) -> float:
    return lib().oracle_e8m0_value(int(s))


def round_bf16(v: float) -> int:
    return int(lib().oracle_round_bf16(float(v)))


def silu(g: float) -> float:
    return lib().oracle_silu(float(g))


def dequant_row(codes, scales, K):
    codes, scales = _c(codes, np.uint8), _c(scales, np.uint8)
    out = np.empty(K, dtype=np.float64)
    lib().oracle_dequant_row(_p(codes), _p(scales), K, _p(out))
    return out


def router_logits(x_bf16, wr_bf16, bias=None):
    x, wr = _c(x_bf16, np.uint16), _c(wr_bf16, np.uint16)
    B, H = x.shape
    E = wr.shape[1]
    b = None if bias is None else _c(bias, np.float32)
    out = np.empty((B, E), dtype=np.float64)
    lib().oracle_router_logits(_p(x), _p(wr), _p(b), B, H, E, _p(out))
    return out


def topk_softmax(logits, k):
    lg = _c(logits, np.float64)
    B, E = lg.shape
    idx = np.empty((B, k), dtype=np.int32)
    w = np.empty((B, k), dtype=np.float64)
    lib().oracle_topk_softmax(_p(lg), B, E, k, _p(idx), _p(w))
    return idx, w


def topk_sigmoid(logits, k, bias=None):
    """Sigmoid scoring: select by sigmoid(l) + bias, weights sigmoid(l) / sum."""
    lg = _c(logits, np.float64)
    B, E = lg.shape
    b = None if bias is None else _c(bias, np.float32)
    idx = np.empty((B, k), dtype=np.int32)
    w = np.empty((B, k), dtype=np.float64)
    lib().oracle_topk_sigmoid(_p(lg), _p(b), B, E, k, _p(idx), _p(w))
    return idx, w


def bucket(topk_idx, E):
    idx = _c(topk_idx, np.int32)
    B, k = idx.shape
    counts = np.empty(E, dtype=np.int32)
    offsets = np.empty(E + 1, dtype=np.int32)
    pair_ids = np.empty(B * k, dtype=np.int32)
    active = np.empty(E, dtype=np.int32)
    n_active = np.empty(1, dtype=np.int32)
    lib().oracle_bucket(_p(idx), B, k, E, _p(counts), _p(offsets), _p(pair_ids), _p(active), _p(n_active))
    na = int(n_active[0])
    return dict(counts=counts, offsets=offsets, pair_ids=pair_ids, active=active[:na].copy(), n_active=na)


def expert_ffn(x, gu_codes, gu_scales, d_codes, d_scales):
    x = _c(x, np.float64)
    H = x.shape[0]
    I = gu_codes.shape[0] // 2
    gc, gs, dc, ds = (_c(a, np.uint8) for a in (gu_codes, gu_scales, d_codes, d_scales))
    h = np.empty(I, dtype=np.float64)
    y = np.empty(H, dtype=np.float64)
    lib().oracle_expert_ffn(_p(x), _p(gc), _p(gs), _p(dc), _p(ds), H, I, _p(h), _p(y))
    return h, y


def shared_ffn(x, gu_bf16, d_bf16):
    x = _c(x, np.float64)
    H = x.shape[0]
    Is = gu_bf16.shape[0] // 2
    gu, d = _c(gu_bf16, np.uint16), _c(d_bf16, np.uint16)
    h = np.empty(Is, dtype=np.float64)
    y = np.empty(H, dtype=np.float64)
    lib().oracle_shared_ffn(_p(x), _p(gu), _p(d), H, Is, _p(h), _p(y))
    return h, y


def layer(x, residual, router_w, router_bias, gu_codes, gu_scales, d_codes, d_scales,
          shared_gu, shared_d, top_k, experts=None, n_threads=1, scoring="softmax", shared_mx=None):
    """Whole layer.  Expert tensors are stacked by slot; `experts` lists the
    expert id of each slot (None: slot i is expert i).  scoring: "softmax"
    (default) or "sigmoid" (bias-corrected selection); shared_mx: MXFP4
    shared expert (gu_codes, gu_scales, d_codes, d_scales) instead of the
    bf16 shared_gu / shared_d.  Returns a dict."""
    x, residual = _c(x, np.uint16), _c(residual, np.uint16)
    wr = _c(router_w, np.uint16)
    B, H = x.shape
    E = wr.shape[1]
    k = int(top_k)
    gc, gs, dc, ds = (_c(a, np.uint8) for a in (gu_codes, gu_scales, d_codes, d_scales))
    I = gc.shape[1] // 2
    sgu = None if shared_gu is None else _c(shared_gu, np.uint16)
    sd = None if shared_d is None else _c(shared_d, np.uint16)
    Is = 0 if sgu is None else sgu.shape[0] // 2
    smx = None
    if shared_mx is not None:
        smx = tuple(_c(a, np.uint8) for a in shared_mx)
        Is = smx[0].shape[0] // 2
        sgu = sd = None
    bias = None if router_bias is None else _c(router_bias, np.float32)
    slot = None
    if experts is not None:
        slot = np.full(E, -1, dtype=np.int32)
        slot[np.asarray(experts, dtype=np.int64)] = np.arange(len(experts), dtype=np.int32)
    r = dict(
        logits=np.empty((B, E)), topk_idx=np.empty((B, k), np.int32), topk_w=np.empty((B, k)),
        counts=np.empty(E, np.int32), offsets=np.empty(E + 1, np.int32),
        pair_ids=np.empty(B * k, np.int32), active=np.empty(E, np.int32),
        n_active=np.empty(1, np.int32), h_routed=np.empty((B * k, I)),
        y_routed=np.empty((B * k, H)), y_shared=np.empty((B, H)), out=np.empty((B, H)),
        out_bf16=np.empty((B, H), np.uint16))
    sc_id = {"softmax": 0, "sigmoid": 1}[scoring]
    mx_ptrs = [None] * 4 if smx is None else [_p(a) for a in smx]
    rc = lib().oracle_layer_v(
        B, H, E, k, I, Is, _p(x), _p(residual), _p(wr), _p(bias), _p(gc), _p(gs), _p(dc), _p(ds),
        _p(slot), _p(sgu), _p(sd), int(n_threads), _p(r["logits"]), _p(r["topk_idx"]),
        _p(r["topk_w"]), _p(r["counts"]), _p(r["offsets"]), _p(r["pair_ids"]), _p(r["active"]),
        _p(r["n_active"]), _p(r["h_routed"]), _p(r["y_routed"]), _p(r["y_shared"]), _p(r["out"]),
        _p(r["out_bf16"]), sc_id, *mx_ptrs)
    if rc != 0:
        raise RuntimeError(f"oracle_layer failed: {rc}")
    na = int(r["n_active"][0])
    r["active"] = r["active"][:na].copy()
    r["n_active"] = na
    return r


def routing(x, router_w, router_bias, top_k, scoring="softmax"):
    """Router, top-k, weights and buckets only (cheap at every size)."""
    if scoring == "sigmoid":
        lg = router_logits(x, router_w, None)
        idx, w = topk_sigmoid(lg, top_k, router_bias)
    else:
        lg = router_logits(x, router_w, router_bias)
        idx, w = topk_softmax(lg, top_k)
    out = bucket(idx, np.asarray(router_w).shape[1])
    out.update(logits=lg, topk_idx=idx, topk_w=w)
    return out
