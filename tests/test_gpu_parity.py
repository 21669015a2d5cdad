"""CUDA path vs the oracle, through the C ABI: routing bit-exact, float
results within the layer's stated tolerance, on the tiny workload (several
batch sizes and edge cases) and the full-size ones."""
import numpy as np
import pytest

import synth
from helpers import W_ABS, Y_MAX_REL, Y_MEAN_REL, Y_ROUTED_MAX_REL, Y_ROUTED_MEAN_REL, bf16_close, metric_close
from gpu_common import (CUDA_CORES, MX, WARP_MMA, assert_routing_equal, create_layer, layer_routing_host,
                        make_device_layer,
                        oracle_layer_for, residual_tokens, routing_buffers, routing_host, routing_struct,
                        to_host_u16)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from sparse_moe_decode_router_b200 import api
    api.load_library()   # fails loudly when the library is not built
    return torch


def run_all_paths(torch, dl, B, max_batch=None, flags=0, token0=0, tiny_every=0):
    """Staged calls, fused forward and host forward on one batch; returns
    GPU results and the oracle's.  tiny_every > 0: activation rows with
    every tiny_every-th element scaled by 2^-30."""
    from sparse_moe_decode_router_b200 import api
    c = dl.cfg
    H, k, E = c.hidden, c.top_k, c.n_experts
    ids = list(range(token0, token0 + B))
    x_h, x_d = dl.tokens(ids, tiny_every=tiny_every)
    r_h, r_d = residual_tokens(c, ids, dl.layer)
    h = create_layer(dl, max_batch or B, flags)
    try:
        rb = routing_buffers(B, k, E)
        rs = routing_struct(rb)
        api.moe_router_topk(h, x_d, B, rs)
        y = torch.full((B * k, H), float("nan"), dtype=torch.float32, device="cuda")
        ys = torch.full((B, H), float("nan"), dtype=torch.float32, device="cuda")
        api.moe_experts_mxfp4(h, x_d, B, rs, y, ys if c.shared_inter else None)
        out_staged = torch.empty((B, H), dtype=torch.bfloat16, device="cuda")
        api.moe_combine_residual(h, B, rs, y, ys if c.shared_inter else None, r_d, out_staged)
        out_fused = torch.empty((B, H), dtype=torch.bfloat16, device="cuda")
        api.moe_layer_forward(h, None, x_d, r_d, out_fused, B)
        xp = torch.from_numpy(x_h.view(np.int16)).pin_memory()
        rp = torch.from_numpy(r_h.view(np.int16)).pin_memory()
        op = torch.empty((B, H), dtype=torch.int16).pin_memory()
        api.moe_layer_forward_host(h, xp, rp, op, B)
        torch.cuda.synchronize()
        assert api.moe_layer_last_device_error(h) == api.MOE_OK
        got = dict(routing=routing_host(rb), y=y.cpu().numpy(), ys=ys.cpu().numpy(),
                   out_staged=to_host_u16(out_staged), out_fused=to_host_u16(out_fused),
                   out_host=op.numpy().view(np.uint16).copy(),
                   fused_routing=layer_routing_host(h, B, k, E))
    finally:
        api.moe_layer_destroy(h)
    ref = oracle_layer_for(dl, x_h, r_h)
    return got, ref


def check_against_oracle(got, ref, shared=True, shared_mx=False):
    """shared_mx: the shared expert is MXFP4 and runs on the MXFP4 streaming
    kernels, so its output gets the routed experts' tolerance."""
    assert_routing_equal(got["routing"], ref, W_ABS)
    assert_routing_equal(got["fused_routing"], ref, W_ABS)
    ok, info = metric_close(got["y"], ref["y_routed"], Y_ROUTED_MAX_REL, Y_ROUTED_MEAN_REL)
    assert ok, f"routed expert outputs: {info}"
    if shared:
        tol = (Y_ROUTED_MAX_REL, Y_ROUTED_MEAN_REL) if shared_mx else (Y_MAX_REL, Y_MEAN_REL)
        ok, info = metric_close(got["ys"], ref["y_shared"], *tol)
        assert ok, f"shared expert output: {info}"
    ok, info = bf16_close(got["out_fused"], ref["out_bf16"])
    assert ok, f"layer output: {info}"
    # the fused path and the staged calls do the same arithmetic in the same order
    assert np.array_equal(got["out_fused"], got["out_staged"])
    assert np.array_equal(got["out_host"], got["out_fused"])


@pytest.fixture(scope="module")
def tiny(torch_cuda):
    return make_device_layer(synth.CONFIGS[0])


@pytest.mark.parametrize("B", [1, 2, 7, 33, 64])
def test_tiny_all_paths_match_oracle(torch_cuda, tiny, B):
    got, ref = run_all_paths(torch_cuda, tiny, B, max_batch=64)
    check_against_oracle(got, ref)


def test_tiny_device_weights_equal_host_generator(torch_cuda, tiny):
    c = tiny.cfg
    host = synth.gen_host_layer(c)
    gc, gs, dc, ds = tiny.host_experts(range(c.n_experts))
    assert np.array_equal(gc, host["gu_codes"]) and np.array_equal(gs, host["gu_scales"])
    assert np.array_equal(dc, host["d_codes"]) and np.array_equal(ds, host["d_scales"])
    assert np.array_equal(tiny.router_w_host, host["router_w"])
    sgu, sd = tiny.host_shared()
    assert np.array_equal(sgu, host["shared_gu"]) and np.array_equal(sd, host["shared_d"])


@pytest.mark.parametrize("variant", ["k1", "k_eq_E", "no_shared", "zipf_bias", "E1024_k32", "I256_H512"])
def test_tiny_variants_match_oracle(torch_cuda, variant):
    base = synth.CONFIGS[0]
    cfg = {"k1": base.with_(top_k=1),
           "k_eq_E": base.with_(top_k=32),
           "no_shared": base.with_(shared_inter=0),
           "zipf_bias": base.with_(zipf_s=1.1, seed=base.seed + 100),
           "E1024_k32": base.with_(n_experts=1024, top_k=32),
           "I256_H512": base.with_(hidden=512, inter=256, shared_inter=64)}[variant]
    if variant == "k_eq_E":
        cfg = cfg.with_(min_gap=0.0)   # every expert is selected: no k+1-th logit
    dl = make_device_layer(cfg)
    for B in (1, 5):
        got, ref = run_all_paths(torch_cuda, dl, B, max_batch=8)
        check_against_oracle(got, ref, shared=cfg.shared_inter > 0)


@pytest.fixture(scope="module")
def skewed_small(torch_cuda):
    # K = 512 and 256 are multiples of 256, so batches above 8 take the grouped
    # tensor-core kernels; the Zipf bias piles tokens onto a few experts
    base = synth.CONFIGS[0]
    return make_device_layer(base.with_(hidden=512, inter=256, shared_inter=64, zipf_s=1.1, seed=base.seed + 300))


@pytest.mark.parametrize("B", [9, 33, 64])
def test_grouped_kernels_match_oracle(torch_cuda, skewed_small, B):
    """Grouped warp-MMA path on every token: B=33 has an expert with 27 tokens
    (four 8-token tiles), B=64 one with 56 (two passes of 32 per item)."""
    got, ref = run_all_paths(torch_cuda, skewed_small, B, max_batch=64, flags=WARP_MMA)
    check_against_oracle(got, ref)
    if B == 64:
        assert ref["counts"].max() > 32


def test_expert_path_selection(torch_cuda, skewed_small):
    """moe_layer_expert_path: batch 1 on the GEMVs and larger batches on
    tcgen05 by default; each selection flag as the header states."""
    from sparse_moe_decode_router_b200 import api
    G, W, T = api.MOE_PATH_GEMV, api.MOE_PATH_GROUPED, api.MOE_PATH_TCGEN05
    want = {0: {1: G, 5: T, 9: T, 64: T}, CUDA_CORES: {1: G, 5: G, 9: G, 64: G},
            WARP_MMA: {1: G, 5: G, 9: W, 64: W}, MX: {1: T, 5: T, 9: T, 64: T}}
    for flags, paths in want.items():
        h = create_layer(skewed_small, 64, flags)
        try:
            assert {B: api.moe_layer_expert_path(h, B) for B in paths} == paths, flags
            with pytest.raises(ValueError):
                api.moe_layer_expert_path(h, 65)
        finally:
            api.moe_layer_destroy(h)


def test_grouped_and_gemv_paths_agree_within_tolerance(torch_cuda, skewed_small):
    """MOE_FLAG_NO_GROUPED keeps batch 64 on the GEMV kernels: the GEMV,
    warp-MMA and tcgen05 paths all meet the oracle (their sums run in
    different fixed orders); the default at batch 64 is tcgen05."""
    got_g, ref = run_all_paths(torch_cuda, skewed_small, 64, max_batch=64, flags=WARP_MMA)
    got_v, _ = run_all_paths(torch_cuda, skewed_small, 64, max_batch=64, flags=CUDA_CORES)
    got_d, _ = run_all_paths(torch_cuda, skewed_small, 64, max_batch=64)
    check_against_oracle(got_d, ref)
    check_against_oracle(got_g, ref)
    check_against_oracle(got_v, ref)


@pytest.mark.parametrize("flags", [1, 2, 4, 7])
def test_tiny_flags_give_identical_results(torch_cuda, tiny, flags):
    base, _ = run_all_paths(torch_cuda, tiny, 3, max_batch=4)
    other, _ = run_all_paths(torch_cuda, tiny, 3, max_batch=4, flags=flags)
    assert np.array_equal(base["out_fused"], other["out_fused"])
    assert np.array_equal(base["y"], other["y"])


def test_layers_of_different_shapes_coexist(torch_cuda, tiny):
    """Kernel instances are shared by every layer in the process: creating a
    layer whose plans need less shared memory must not break the launches of
    a larger layer created before it."""
    from sparse_moe_decode_router_b200 import api
    torch = torch_cuda
    base = synth.CONFIGS[0]
    big = make_device_layer(base.with_(hidden=512, inter=256, shared_inter=64))
    hb = create_layer(big, 8)
    hs = create_layer(tiny, 8)
    try:
        for dl, h in ((big, hb), (tiny, hs), (big, hb)):
            c = dl.cfg
            for B in (1, 5):
                ids = list(range(B))
                x_h, x_d = dl.tokens(ids)
                r_h, r_d = residual_tokens(c, ids, dl.layer)
                out = torch.empty((B, c.hidden), dtype=torch.bfloat16, device="cuda")
                api.moe_layer_forward(h, None, x_d, r_d, out, B)
                torch.cuda.synchronize()
                assert api.moe_layer_last_device_error(h) == api.MOE_OK
                ref = oracle_layer_for(dl, x_h, r_h)
                assert_routing_equal(layer_routing_host(h, B, c.top_k, c.n_experts), ref, W_ABS)
                ok, info = bf16_close(to_host_u16(out), ref["out_bf16"])
                assert ok, (c.hidden, B, info)
    finally:
        api.moe_layer_destroy(hs)
        api.moe_layer_destroy(hb)


def test_invalid_calls_are_rejected(torch_cuda, tiny):
    from sparse_moe_decode_router_b200 import api
    torch = torch_cuda
    h = create_layer(tiny, 4)
    try:
        x = torch.zeros((8, tiny.cfg.hidden), dtype=torch.bfloat16, device="cuda")
        out = torch.zeros_like(x)
        for B in (0, 5, -1):
            with pytest.raises(api.MoEError) as e:
                api.moe_layer_forward(h, None, x, x, out, B)
            assert e.value.status == api.MOE_ERR_INVALID_ARG
        with pytest.raises(api.MoEError):
            api.moe_layer_forward(h, None, x.data_ptr() + 2, x, out, 1)   # misaligned
        with pytest.raises(api.MoEError):
            api.moe_experts_mxfp4(h, x, 1, None, None, None)
    finally:
        api.moe_layer_destroy(h)


# ----------------------------------------------------------- full size -----
@pytest.fixture(scope="module")
def full_layers(torch_cuda):
    cache = {}

    def get(i):
        if i not in cache:
            cache.clear()
            torch_cuda.cuda.empty_cache()
            cache[i] = make_device_layer(synth.CONFIGS[i])
        return cache[i]
    yield get
    cache.clear()


@pytest.mark.parametrize("cfg_id,flags", [(1, 0), (2, 0), (2, CUDA_CORES)],
                         ids=["b1", "b8_default", "b8_cuda_cores"])
def test_full_size_matches_oracle(torch_cuda, full_layers, cfg_id, flags):
    """Batch 1 (CUDA-core GEMVs by default) and batch 8 (tcgen05 by default,
    and on the GEMVs)."""
    dl = full_layers(cfg_id)
    got, ref = run_all_paths(torch_cuda, dl, dl.cfg.batch, flags=flags)
    check_against_oracle(got, ref)
    if cfg_id == 2:
        assert 100 <= ref["n_active"] <= 128


def test_full_size_b64_zipf(torch_cuda, full_layers):
    """Batch 64 with the Zipf-skewed router on the grouped warp-MMA kernels
    (the tcgen05 kernels, the default there, have their own test below):
    routing of all 64 tokens bit-exact, layer outputs of a sample of tokens
    against the oracle run on those tokens (tokens are independent)."""
    from sparse_moe_decode_router_b200 import api
    import oracle
    torch = torch_cuda
    dl = full_layers(3)
    c = dl.cfg
    B, H, k, E = c.batch, c.hidden, c.top_k, c.n_experts
    ids = list(range(B))
    x_h, x_d = dl.tokens(ids)
    r_h, r_d = residual_tokens(c, ids)
    ref_rt = oracle.routing(x_h, dl.router_w_host, dl.bias_host, k)
    assert ref_rt["n_active"] > 300 and ref_rt["counts"].max() >= 8   # skewed: hot experts
    h = create_layer(dl, B, WARP_MMA)
    try:
        out = torch.empty((B, H), dtype=torch.bfloat16, device="cuda")
        api.moe_layer_forward(h, None, x_d, r_d, out, B)
        torch.cuda.synchronize()
        got_rt = layer_routing_host(h, B, k, E)
        out_h = to_host_u16(out)
        out2 = torch.empty_like(out)
        api.moe_layer_forward(h, None, x_d, r_d, out2, B)
        torch.cuda.synchronize()
        assert api.moe_layer_last_device_error(h) == api.MOE_OK
        assert np.array_equal(to_host_u16(out2), out_h)          # run to run bit-identical
    finally:
        api.moe_layer_destroy(h)
    assert_routing_equal(got_rt, ref_rt, W_ABS)
    # hottest expert's tokens plus a spread of others
    hot = int(np.argmax(ref_rt["counts"]))
    hot_tokens = sorted(set(np.nonzero((ref_rt["topk_idx"] == hot).any(1))[0].tolist()))
    sample = sorted(set(hot_tokens[:3] + [0, 21, 42, 63]))
    ref = oracle_layer_for(dl, x_h[sample], r_h[sample])
    ok, info = bf16_close(out_h[sample], ref["out_bf16"])
    assert ok, info


def test_full_b1_run_to_run_bit_identical(torch_cuda, full_layers):
    from sparse_moe_decode_router_b200 import api
    torch = torch_cuda
    dl = full_layers(1)
    x_h, x_d = dl.tokens([5])
    r_h, r_d = residual_tokens(dl.cfg, [5])
    h = create_layer(dl, 1)
    try:
        outs = []
        for _ in range(20):
            o = torch.empty((1, dl.cfg.hidden), dtype=torch.bfloat16, device="cuda")
            api.moe_layer_forward(h, None, x_d, r_d, o, 1)
            outs.append(o)
        torch.cuda.synchronize()
        first = to_host_u16(outs[0])
        for o in outs[1:]:
            assert np.array_equal(to_host_u16(o), first)
    finally:
        api.moe_layer_destroy(h)


# ------------------------------------------- tcgen05 block-scaled path -----


@pytest.mark.parametrize("B", [1, 2, 7, 33, 64])
def test_mx_tiny_all_paths_match_oracle(torch_cuda, tiny, B):
    """Routed experts on the tcgen05 kernels (E2M1 weights x E2M1 activation
    terms, E8M0 scales on both operands): tiny layer, one 128-row tile per
    projection; the down projection's K (128) is half a pipeline stage."""
    got, ref = run_all_paths(torch_cuda, tiny, B, max_batch=64, flags=MX)
    check_against_oracle(got, ref)


@pytest.mark.parametrize("B", [1, 5, 9, 33, 64])
def test_mx_skewed_matches_oracle(torch_cuda, skewed_small, B):
    """Several K stages and row tiles; B = 64 has an expert with 56 tokens
    (four passes of up to 16 tokens over its weights)."""
    got, ref = run_all_paths(torch_cuda, skewed_small, B, max_batch=64, flags=MX)
    check_against_oracle(got, ref)


@pytest.mark.parametrize("B", [1, 9, 33])
def test_mx_weights_as_a_kernel_matches_oracle(torch_cuda, B):
    """Hidden 384 (a multiple of 128, not of 256): the tcgen05 path keeps the
    kernels with the weights as the A operand (128-row tiles of one
    projection, activation terms as N columns)."""
    base = synth.CONFIGS[0]
    dl = make_device_layer(base.with_(hidden=384, inter=256, shared_inter=64, seed=base.seed + 700))
    got, ref = run_all_paths(torch_cuda, dl, B, max_batch=64, flags=MX)
    check_against_oracle(got, ref)


def test_mx_and_gemv_paths_agree(torch_cuda, skewed_small):
    got_m, ref = run_all_paths(torch_cuda, skewed_small, 7, max_batch=8, flags=MX)
    got_g, _ = run_all_paths(torch_cuda, skewed_small, 7, max_batch=8)
    check_against_oracle(got_m, ref)
    check_against_oracle(got_g, ref)
    assert np.array_equal(got_m["routing"]["topk_idx"], got_g["routing"]["topk_idx"])


@pytest.mark.parametrize("cfg_id", [1, 2])
def test_mx_full_size_matches_oracle(torch_cuda, full_layers, cfg_id):
    dl = full_layers(cfg_id)
    got, ref = run_all_paths(torch_cuda, dl, dl.cfg.batch, flags=MX)
    check_against_oracle(got, ref)


def test_mx_full_size_b64_zipf(torch_cuda, full_layers):
    """Batch 64, Zipf-skewed routing, tcgen05 path: routing of all 64 tokens
    bit-exact; routed expert outputs (staged call) and layer outputs (fused
    call) of a sample of tokens, the hottest expert's among them, against the
    oracle run on those tokens (tokens are independent of each other)."""
    from sparse_moe_decode_router_b200 import api
    import oracle
    torch = torch_cuda
    dl = full_layers(3)
    c = dl.cfg
    B, H, k, E = c.batch, c.hidden, c.top_k, c.n_experts
    ids = list(range(B))
    x_h, x_d = dl.tokens(ids)
    r_h, r_d = residual_tokens(c, ids)
    ref_rt = oracle.routing(x_h, dl.router_w_host, dl.bias_host, k)
    h = create_layer(dl, B, MX)
    try:
        out = torch.empty((B, H), dtype=torch.bfloat16, device="cuda")
        api.moe_layer_forward(h, None, x_d, r_d, out, B)
        y = torch.empty((B * k, H), dtype=torch.float32, device="cuda")
        ys = torch.empty((B, H), dtype=torch.float32, device="cuda")
        api.moe_experts_mxfp4(h, x_d, B, None, y, ys)
        torch.cuda.synchronize()
        assert api.moe_layer_last_device_error(h) == api.MOE_OK
        got_rt = layer_routing_host(h, B, k, E)
        out_h, y_h = to_host_u16(out), y.cpu().numpy()
    finally:
        api.moe_layer_destroy(h)
    assert_routing_equal(got_rt, ref_rt, W_ABS)
    hot = int(np.argmax(ref_rt["counts"]))
    hot_tokens = sorted(set(np.nonzero((ref_rt["topk_idx"] == hot).any(1))[0].tolist()))
    sample = sorted(set(hot_tokens[:3] + [0, 21, 42, 63]))
    ref = oracle_layer_for(dl, x_h[sample], r_h[sample])
    ok, info = bf16_close(out_h[sample], ref["out_bf16"])
    assert ok, info
    rows = np.concatenate([np.arange(b * k, (b + 1) * k) for b in sample])
    ok, info = metric_close(y_h[rows], ref["y_routed"], Y_ROUTED_MAX_REL, Y_ROUTED_MEAN_REL)
    assert ok, info


@pytest.mark.parametrize("flags", [CUDA_CORES, MX], ids=["cuda_cores", "tcgen05"])
def test_full_size_verify_b8_matches_oracle(torch_cuda, full_layers, flags):
    """Speculative-decoding verify shape: 8 positions of one sequence whose
    activations share most of their direction, so they route to far fewer
    distinct experts than 8 independent tokens (about 40 of 128)."""
    dl = full_layers(5)
    got, ref = run_all_paths(torch_cuda, dl, 8, flags=flags)
    check_against_oracle(got, ref)
    assert ref["n_active"] < 64
