"""The persistent single-launch batch-1 layer (MOE_FLAG_PERSISTENT): one
cooperative kernel runs the router (with the shared expert's gate/up rows
and the routing finish), the shared down projection, the routed experts and
the combine, with in-kernel grid barriers in between.  It must match the
oracle, and the chained kernels bit for bit (same arithmetic per stream),
also inside a CUDA graph."""
import numpy as np
import pytest

import synth
from gpu_common import create_layer, layer_routing_host, make_device_layer, oracle_layer_for, residual_tokens, to_host_u16
from helpers import W_ABS, bf16_close
from gpu_common import assert_routing_equal

pytestmark = pytest.mark.gpu

PERSISTENT = 0x40


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from sparse_moe_decode_router_b200 import api
    api.load_library()
    return torch


def _forward(torch, h, dl, ids):
    from sparse_moe_decode_router_b200 import api
    c = dl.cfg
    B = len(ids)
    x_h, x_d = dl.tokens(ids)
    r_h, r_d = residual_tokens(c, ids, dl.layer)
    out = torch.empty((B, c.hidden), dtype=torch.bfloat16, device="cuda")
    api.moe_layer_forward(h, None, x_d, r_d, out, B)
    torch.cuda.synchronize()
    assert api.moe_layer_last_device_error(h) == api.MOE_OK
    return x_h, r_h, to_host_u16(out)


@pytest.mark.parametrize("cfg_id", [0, 1])
def test_persistent_matches_oracle_and_chain(torch_cuda, cfg_id):
    from sparse_moe_decode_router_b200 import api
    torch = torch_cuda
    dl = make_device_layer(synth.CONFIGS[cfg_id])
    c = dl.cfg
    hp = create_layer(dl, 4, PERSISTENT)
    hc = create_layer(dl, 4)
    try:
        for t in range(3):
            x_h, r_h, got = _forward(torch, hp, dl, [t])
            _, _, chain = _forward(torch, hc, dl, [t])
            ref = oracle_layer_for(dl, x_h, r_h)
            assert_routing_equal(layer_routing_host(hp, 1, c.top_k, c.n_experts), ref, W_ABS)
            ok, info = bf16_close(got, ref["out_bf16"])
            assert ok, info
            assert np.array_equal(got, chain)
        # batches above one take the chained kernels on the same layer
        x_h, r_h, got = _forward(torch, hp, dl, [10, 11, 12])
        ok, info = bf16_close(got, oracle_layer_for(dl, x_h, r_h)["out_bf16"])
        assert ok, info
    finally:
        api.moe_layer_destroy(hp)
        api.moe_layer_destroy(hc)
        del dl
        torch.cuda.empty_cache()


def test_persistent_in_a_graph_two_layers(torch_cuda):
    """Two full-size layers chained through the residual, 8 decode steps in
    one CUDA graph: the persistent kernels against the chained kernels."""
    from sparse_moe_decode_router_b200 import api
    torch = torch_cuda
    cfg = synth.CONFIGS[4]
    layers = [make_device_layer(cfg, l) for l in range(2)]
    n_steps, H = 8, cfg.hidden
    xs = []
    for l in range(2):
        _, xd = layers[l].tokens(range(n_steps))
        xs.append(xd)
    _, r0 = residual_tokens(cfg, range(n_steps), 0)
    results = {}
    for flags in (0, PERSISTENT):
        hs = [create_layer(dl, 1, flags) for dl in layers]
        try:
            outs = [[torch.empty((1, H), dtype=torch.bfloat16, device="cuda") for _ in range(2)] for _ in range(n_steps)]
            g = torch.cuda.CUDAGraph()
            s = torch.cuda.Stream()
            s.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(s):
                with torch.cuda.graph(g, stream=s):
                    for t in range(n_steps):
                        res = r0[t:t + 1]
                        for l in range(2):
                            api.moe_layer_forward(hs[l], hs[(l + 1) % 2], xs[l][t:t + 1], res, outs[t][l], 1,
                                                  stream=torch.cuda.current_stream())
                            res = outs[t][l]
            g.replay()
            torch.cuda.synchronize()
            for hd in hs:
                assert api.moe_layer_last_device_error(hd) == api.MOE_OK
            results[flags] = [[to_host_u16(outs[t][l]) for l in range(2)] for t in range(n_steps)]
            del g
        finally:
            for hd in hs:
                api.moe_layer_destroy(hd)
    for t in range(n_steps):
        for l in range(2):
            assert np.array_equal(results[PERSISTENT][t][l], results[0][t][l]), (t, l)


def test_persistent_refuses_unsupported_combinations(torch_cuda):
    from sparse_moe_decode_router_b200 import api
    base = synth.CONFIGS[0]
    for cfg, flags in ((base, PERSISTENT | 0x2), (base.with_(shared_format="mxfp4"), PERSISTENT),
                       (base.with_(inter=2048), PERSISTENT)):
        dl = make_device_layer(cfg)
        with pytest.raises(api.MoEError) as e:
            create_layer(dl, 1, flags)
        assert e.value.status == api.MOE_ERR_UNSUPPORTED
