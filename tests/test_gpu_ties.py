"""Deterministic top-k under exact ties, through the C ABI.

Integer router weights, bias and activations make every logit an integer,
exact in the kernel's fp32 and in the oracle's fp64, so both sides take the
top-k decision on identical values.  The router columns come in groups of
identical copies scattered over the expert ids, so many selections have to
break ties: of equal logits the lower expert id is selected.  Routing must
match the oracle bit for bit, through a layer's router call and through the
allocation-free entry, at the top-k kernel's three slice layouts."""
import dataclasses

import numpy as np
import pytest

import oracle
import synth
from gpu_common import assert_routing_equal, create_layer, make_device_layer, routing_buffers, routing_host, routing_struct
from helpers import TIE_SHAPES, W_ABS
from synth.workload import u16_to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("E,k,copies", TIE_SHAPES)
@pytest.mark.parametrize("with_bias", [True, False])
def test_equal_logits_go_to_the_lower_expert_id(E, k, copies, with_bias):
    import torch
    from sparse_moe_decode_router_b200 import api
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    api.load_library()
    cfg = synth.CONFIGS[0].with_(n_experts=E, top_k=k)
    wr, bias, _ = synth.gen_tied_router(cfg, n_copies=copies, with_bias=with_bias)
    dl = make_device_layer(cfg)
    bias_d = None if bias is None else torch.from_numpy(bias).to("cuda")
    dl = dataclasses.replace(dl, router_w=u16_to_device(wr), router_bias=bias_d, router_w_host=wr,
                             bias_host=bias)
    w_em = dl.router_w.t().contiguous()          # expert-major copy for the allocation-free entry
    x_all = synth.gen_tied_tokens(cfg, 64)
    h = create_layer(dl, 64)
    try:
        for B in (1, 7, 64):
            x_h = np.ascontiguousarray(x_all[:B])
            x_d = u16_to_device(x_h)
            ref = oracle.routing(x_h, wr, bias, k)
            srt = -np.sort(-ref["logits"], axis=1)
            if B > 1:   # the case really breaks ties at the selection boundary
                assert np.any(srt[:, k - 1] == srt[:, k])
            got = routing_buffers(B, k, E)
            api.moe_router_topk(h, x_d, B, routing_struct(got))
            got_na = routing_buffers(B, k, E)
            api.moe_router_topk_noalloc(w_em, bias_d, cfg.hidden, E, k, x_d, B, routing_struct(got_na))
            torch.cuda.synchronize()
            assert api.moe_layer_last_device_error(h) == api.MOE_OK
            assert api.moe_router_topk_noalloc_last_error() == api.MOE_OK
            assert_routing_equal(routing_host(got), ref, W_ABS)
            assert_routing_equal(routing_host(got_na), ref, W_ABS)
    finally:
        api.moe_layer_destroy(h)
