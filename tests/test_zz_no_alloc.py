"""The allocation-free router entry point (moe_router_topk_noalloc).

It serves callers that cannot allocate device memory (an engine that has
reserved the GPU's memory up front, a framework that must account for every
device byte).  Its scratch is a fixed array inside the library, shared by all
calls, so the check runs two calls in a row with different inputs: each must
reproduce what the allocating entry point (moe_router_topk on a layer)
returns for the same inputs.  The layers here are created with
MOE_FLAG_NO_GROUPED so that their router runs the same CUDA-core kernel at
every batch size (above batch 1 the default path computes the logits on the
tensor cores, in another summation order: the same selection, weights equal
to fp32 rounding).  This file sorts last so that a run stopping at the first
failure has already run every other test."""
import numpy as np
import pytest

import synth
from gpu_common import CUDA_CORES, create_layer, make_device_layer, routing_buffers, routing_host, routing_struct

pytestmark = pytest.mark.gpu


def test_noalloc_router_matches_layer_router_twice():
    import torch
    from sparse_moe_decode_router_b200 import api
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    api.load_library()
    cfg = synth.CONFIGS[0].with_(zipf_s=1.1, seed=synth.CONFIGS[0].seed + 7)   # with a router bias
    dl = make_device_layer(cfg)
    H, E, k = cfg.hidden, cfg.n_experts, cfg.top_k
    w_em = dl.router_w.t().contiguous()          # expert-major copy, made by the caller
    h = create_layer(dl, 64, CUDA_CORES)
    try:
        for call, B in enumerate((5, 64)):
            _, x = dl.tokens(range(100 * call, 100 * call + B))
            want = routing_buffers(B, k, E)
            api.moe_router_topk(h, x, B, routing_struct(want))
            got = routing_buffers(B, k, E)
            api.moe_router_topk_noalloc(w_em, dl.router_bias, H, E, k, x, B, routing_struct(got))
            torch.cuda.synchronize()
            assert api.moe_router_topk_noalloc_last_error() == api.MOE_OK
            g, w = routing_host(got), routing_host(want)
            for key in ("topk_idx", "counts", "offsets", "pair_ids", "active"):
                assert np.array_equal(g[key], w[key]), (call, key)
            assert g["n_active"] == w["n_active"]
            assert np.array_equal(g["topk_w"], w["topk_w"]), call   # same kernels: bit-identical
        # sizes beyond the fixed scratch are refused, nothing launched
        with pytest.raises(api.MoEError) as e:
            api.moe_router_topk_noalloc(w_em, None, H, E, k, x, 65, routing_struct(routing_buffers(1, k, E)))
        assert e.value.status == api.MOE_ERR_INVALID_ARG
    finally:
        api.moe_layer_destroy(h)


@pytest.mark.parametrize("cfg_id,batches", [(1, (1,)), (3, (1, 64))])
def test_noalloc_router_full_size_matches_oracle_and_layer(cfg_id, batches):
    """Full-size router (hidden 7168, 896 experts, top-16; config 3 adds its
    Zipf bias): the allocation-free entry against the oracle (indices,
    counts, offsets, pairs and active list exactly, weights within the
    routing tolerance) and against the layer's router, whose batch-1 call
    runs a kernel instance specialised for hidden 7168, bit for bit."""
    import torch
    import oracle
    from helpers import W_ABS
    from gpu_common import assert_routing_equal
    from sparse_moe_decode_router_b200 import api
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    api.load_library()
    cfg = synth.CONFIGS[cfg_id]
    dl = make_device_layer(cfg)
    H, E, k = cfg.hidden, cfg.n_experts, cfg.top_k
    w_em = dl.router_w.t().contiguous()
    h = create_layer(dl, max(batches), CUDA_CORES)
    try:
        for B in batches:
            x_h, x = dl.tokens(range(B))
            want = routing_buffers(B, k, E)
            api.moe_router_topk(h, x, B, routing_struct(want))
            got = routing_buffers(B, k, E)
            api.moe_router_topk_noalloc(w_em, dl.router_bias, H, E, k, x, B, routing_struct(got))
            torch.cuda.synchronize()
            assert api.moe_router_topk_noalloc_last_error() == api.MOE_OK
            assert api.moe_layer_last_device_error(h) == api.MOE_OK
            g, w = routing_host(got), routing_host(want)
            ref = oracle.routing(x_h, dl.router_w_host, dl.bias_host, k)
            assert_routing_equal(g, ref, W_ABS)
            for key in ("topk_idx", "counts", "offsets", "pair_ids", "active"):
                assert np.array_equal(g[key], w[key]), (B, key)
            assert np.array_equal(g["topk_w"], w["topk_w"]), B
    finally:
        api.moe_layer_destroy(h)
        del dl, w_em
        torch.cuda.empty_cache()
