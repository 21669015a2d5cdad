"""GPU-test plumbing: device workloads, routing buffers, oracle runs."""
import os

import numpy as np

import oracle
from synth.workload import make_device_layer, residual_tokens, to_host_u16


def torch():
    import torch as t
    return t


class DevPtr:
    """Wrap a raw device pointer as a torch tensor (via __cuda_array_interface__)."""

    def __init__(self, ptr, shape, typestr):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr,
                                         "data": (int(ptr), False), "version": 3}


def view_device(ptr, shape, typestr):
    return torch().as_tensor(DevPtr(ptr, shape, typestr), device="cuda")


# MOE_FLAG_* selecting the routed-expert kernels (the default: batch 1 on the
# CUDA-core GEMVs, larger batches on tcgen05)
CUDA_CORES = 0x8   # MOE_FLAG_NO_GROUPED: the GEMVs at every batch size
MX = 0x10          # MOE_FLAG_MX_EXPERTS: tcgen05 at every batch size
WARP_MMA = 0x80    # MOE_FLAG_WARP_MMA: grouped warp-level MMA above batch 8


def create_layer(dl, max_batch, flags=0):
    from sparse_moe_decode_router_b200 import api
    c = dl.cfg
    cfg = api.moe_layer_config(c.hidden, c.n_experts, c.top_k, c.inter, c.shared_inter, max_batch, flags)
    return api.moe_layer_create(cfg, dl.weights_struct())


def routing_buffers(B, k, E):
    t = torch()
    d = dict(topk_idx=t.full((B, k), -7, dtype=t.int32, device="cuda"),
             topk_w=t.full((B, k), -1.0, dtype=t.float32, device="cuda"),
             counts=t.full((E,), -7, dtype=t.int32, device="cuda"),
             offsets=t.full((E + 1,), -7, dtype=t.int32, device="cuda"),
             pair_ids=t.full((B * k,), -7, dtype=t.int32, device="cuda"),
             active=t.full((E,), -7, dtype=t.int32, device="cuda"),
             n_active=t.full((1,), -7, dtype=t.int32, device="cuda"))
    return d


def routing_struct(d):
    from sparse_moe_decode_router_b200 import api
    return api.make_routing(d["topk_idx"], d["topk_w"], d["counts"], d["offsets"], d["pair_ids"],
                            d["active"], d["n_active"])


def layer_routing_host(handle, B, k, E):
    """The layer's own routing plan (after moe_layer_forward), copied to the host."""
    from sparse_moe_decode_router_b200 import api
    r = api.moe_layer_routing(handle)
    na = int(view_device(r.n_active, (1,), "<i4").cpu()[0])
    return dict(topk_idx=view_device(r.topk_idx, (B, k), "<i4").cpu().numpy(),
                topk_w=view_device(r.topk_w, (B, k), "<f4").cpu().numpy(),
                counts=view_device(r.counts, (E,), "<i4").cpu().numpy(),
                offsets=view_device(r.offsets, (E + 1,), "<i4").cpu().numpy(),
                pair_ids=view_device(r.pair_ids, (B * k,), "<i4").cpu().numpy(),
                active=view_device(r.active, (E,), "<i4").cpu().numpy()[:na], n_active=na)


def routing_host(d):
    na = int(d["n_active"].cpu()[0])
    out = {k: v.cpu().numpy() for k, v in d.items() if k != "n_active"}
    out["active"] = out["active"][:na]
    out["n_active"] = na
    return out


def assert_routing_equal(got, ref, w_abs):
    assert np.array_equal(got["topk_idx"], ref["topk_idx"]), "top-k indices differ"
    assert got["n_active"] == ref["n_active"]
    for key in ("counts", "offsets", "pair_ids", "active"):
        assert np.array_equal(got[key], ref[key]), f"{key} differs"
    dw = np.abs(got["topk_w"].astype(np.float64) - ref["topk_w"]).max()
    assert dw <= w_abs, f"routing weights differ by {dw}"


def oracle_threads():
    return max(1, min(64, os.cpu_count() or 1))


def oracle_layer_for(dl, x_host, res_host):
    """The oracle on a device workload: routing first, then only the experts it selects."""
    c = dl.cfg
    rt = oracle.routing(x_host, dl.router_w_host, dl.bias_host, c.top_k, scoring=c.scoring)
    sel = np.unique(rt["topk_idx"])
    gc, gs, dc, ds = dl.host_experts(sel)
    sgu, sd = dl.host_shared() if c.shared_inter > 0 else (None, None)
    return oracle.layer(x_host, res_host, dl.router_w_host, dl.bias_host, gc, gs, dc, ds, sgu, sd, c.top_k,
                        experts=sel, n_threads=oracle_threads(), scoring=c.scoring,
                        shared_mx=dl.host_shared_mx())


__all__ = ["make_device_layer", "residual_tokens", "to_host_u16"]
