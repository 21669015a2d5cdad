"""Four full-size layers chained through the residual, batch 1, 64 decode
steps captured in one CUDA graph (programmatic dependent launch inside,
next-layer L2 prefetch on).  Each step is a new token: its residual stream
starts from that token's seeded residual and passes through the four layers
(out of layer l is the residual of layer l+1).  Every layer-step output is
checked against the oracle run on its own chain."""
import numpy as np
import pytest

import oracle
import synth
from helpers import bf16_close
from gpu_common import create_layer, make_device_layer, oracle_threads, residual_tokens, to_host_u16

pytestmark = pytest.mark.gpu


def build_stack_graph(torch, layers, handles, xs, r0s, n_steps):
    """Capture n_steps x n_layers moe_layer_forward calls into one graph
    (step t starts from residual r0s[t]).  Returns (graph, outs[t][l])."""
    from sparse_moe_decode_router_b200 import api
    nl = len(handles)
    H = layers[0].cfg.hidden
    outs = [[torch.empty((1, H), dtype=torch.bfloat16, device="cuda") for _ in range(nl)] for _ in range(n_steps)]
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        # one eager pass outside capture is not needed: the library allocates nothing per call
        with torch.cuda.graph(g, stream=s):
            for t in range(n_steps):
                res = r0s[t]
                for l in range(nl):
                    nxt = handles[(l + 1) % nl]
                    api.moe_layer_forward(handles[l], nxt, xs[t][l], res, outs[t][l], 1,
                                          stream=torch.cuda.current_stream())
                    res = outs[t][l]
    return g, outs


def test_stack4_graph_64_steps_every_step_matches_oracle():
    import torch
    from sparse_moe_decode_router_b200 import api
    cfg = synth.CONFIGS[4]
    nl, n_steps, H, k = cfg.n_layers, cfg.n_steps, cfg.hidden, cfg.top_k
    layers = [make_device_layer(cfg, l) for l in range(nl)]
    x_host = [[None] * nl for _ in range(n_steps)]
    xs = [[None] * nl for _ in range(n_steps)]
    for l in range(nl):
        xh, xd = layers[l].tokens(range(n_steps))     # token id = step, layer-specific substream
        for t in range(n_steps):
            x_host[t][l] = xh[t:t + 1]
            xs[t][l] = xd[t:t + 1]
    r0_h, r0_d = residual_tokens(cfg, range(n_steps), 0)   # one fresh residual per step (token)
    r0s = [r0_d[t:t + 1] for t in range(n_steps)]
    handles = [create_layer(dl, 1) for dl in layers]
    try:
        g, outs = build_stack_graph(torch, layers, handles, xs, r0s, n_steps)
        g.replay()
        torch.cuda.synchronize()
        for hd in handles:
            assert api.moe_layer_last_device_error(hd) == api.MOE_OK
        got = [[to_host_u16(outs[t][l]) for l in range(nl)] for t in range(n_steps)]
        # replay again: bit-identical
        g.replay()
        torch.cuda.synchronize()
        assert all(np.array_equal(to_host_u16(outs[t][l]), got[t][l]) for t in range(n_steps) for l in range(nl))
        del g
    finally:
        for hd in handles:
            api.moe_layer_destroy(hd)
    shared = [dl.host_shared() for dl in layers]
    worst = 0.0
    for t in range(n_steps):
        res = r0_h[t:t + 1]
        for l in range(nl):
            dl = layers[l]
            rt = oracle.routing(x_host[t][l], dl.router_w_host, None, k)
            sel = np.unique(rt["topk_idx"])
            gc, gs, dc, ds = dl.host_experts(sel)
            ref = oracle.layer(x_host[t][l], res, dl.router_w_host, None, gc, gs, dc, ds, shared[l][0], shared[l][1],
                               k, experts=sel, n_threads=oracle_threads())
            ok, info = bf16_close(got[t][l], ref["out_bf16"])
            assert ok, (t, l, info)
            worst = max(worst, info["mean_rel"])
            res = ref["out_bf16"]        # the oracle chains its own outputs
    print(f"stack: worst mean relative error {worst:.2e}")
