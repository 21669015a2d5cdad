"""CUDA path vs the oracle where the MXFP4 format and the launch chain have
their corners.

* Corner-case expert weights (synth.gen_edge_mxfp4): every 32-element block
  holds all 16 E2M1 codes (negative zero included), scale bytes spread over
  2^-40 .. 2^12 (gate/up) and 2^-12 .. 2^40 (down) with a share of s = 0
  blocks (2^-127), and activation rows that mix elements 2^30 apart.  The
  kernels' range-dependent steps (power-of-two staging of the activations,
  bounded f16 partial sums, the fp32 scale multiply after the block sum, the
  E8M0 decode of s = 0) all meet values far from the synthetic band.  Both
  expert paths run: the streaming GEMV kernels (batches up to 8) and the
  grouped tensor-core kernels (larger batches, K a multiple of 256).
* The full-size layer with every scale byte shifted by +-20 from the
  generator's band.
* Ordering under programmatic dependent launch: the layer's x and residual
  are written by a kernel launched on the same stream just before the layer,
  inside one CUDA graph, and the source changes before every replay.  A
  kernel that read x before its dependency wait (the decode-path pages'
  compiler-hoisting bug: yeyulingfeng, section 03) would see the previous
  replay's token and fail the comparison."""
import numpy as np
import pytest

import oracle
import synth
from gpu_common import (assert_routing_equal, create_layer, layer_routing_host, make_device_layer,
                        oracle_layer_for, residual_tokens, to_host_u16)
from helpers import W_ABS, bf16_close
from synth.workload import with_edge_experts
from test_gpu_parity import check_against_oracle, run_all_paths

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    from sparse_moe_decode_router_b200 import api
    api.load_library()
    return torch


@pytest.fixture(scope="module")
def edge_tiny(torch_cuda):
    return with_edge_experts(make_device_layer(synth.CONFIGS[0]))


@pytest.fixture(scope="module")
def edge_medium(torch_cuda):
    base = synth.CONFIGS[0]
    cfg = base.with_(hidden=512, inter=256, shared_inter=64, zipf_s=1.1, seed=base.seed + 300)
    return with_edge_experts(make_device_layer(cfg))


def _check_edge_weights(dl):
    gc, gs, dc, ds = dl.host_experts(range(dl.cfg.n_experts))
    for codes in (gc, dc):
        nib = np.stack([codes & 15, codes >> 4], -1).reshape(-1, 32)
        assert all((np.bincount(b, minlength=16) == 2).all() for b in nib[:64])
    assert (gs == 0).any() and gs[gs > 0].min() <= 88 and gs.max() >= 138
    assert (ds == 0).any() and ds[ds > 0].min() <= 116 and ds.max() >= 166


@pytest.mark.parametrize("flags", [0x8, 0x10], ids=["cuda_cores", "tcgen05"])
@pytest.mark.parametrize("B", [1, 2, 7])
def test_edge_mxfp4_gemv_path_matches_oracle(torch_cuda, edge_tiny, B, flags):
    _check_edge_weights(edge_tiny)
    got, ref = run_all_paths(torch_cuda, edge_tiny, B, max_batch=8, tiny_every=7, flags=flags)
    assert np.abs(ref["y_routed"]).max() > 1e18           # the wide scales reach the outputs
    check_against_oracle(got, ref)


@pytest.mark.parametrize("flags", [0x80, 0x10], ids=["cuda_cores_warp_mma", "tcgen05"])
@pytest.mark.parametrize("B", [5, 9, 33])
def test_edge_mxfp4_grouped_and_gemv_paths_match_oracle(torch_cuda, edge_medium, B, flags):
    """With MOE_FLAG_WARP_MMA, B = 5 stays on the GEMV kernels and 9, 33 take
    the grouped warp-MMA kernels; with MOE_FLAG_MX_EXPERTS, all run on tcgen05."""
    _check_edge_weights(edge_medium)
    got, ref = run_all_paths(torch_cuda, edge_medium, B, max_batch=64, tiny_every=7, flags=flags)
    check_against_oracle(got, ref)


@pytest.mark.parametrize("shift", [(20, -20), (-20, 20)])
def test_full_size_shifted_scales_match_oracle(torch_cuda, shift):
    """Every E8M0 byte of the full-size layer moved by +-20 (gate/up, down)."""
    torch = torch_cuda
    dl = make_device_layer(synth.CONFIGS[1])
    try:
        lo = min(int(dl.gu_scales.min()), int(dl.d_scales.min()))
        hi = max(int(dl.gu_scales.max()), int(dl.d_scales.max()))
        assert lo - 20 >= 1 and hi + 20 <= 254
        dl.gu_scales.add_(shift[0])
        dl.d_scales.add_(shift[1])
        torch.cuda.synchronize()
        got, ref = run_all_paths(torch, dl, 1)
        check_against_oracle(got, ref)
    finally:
        del dl
        torch.cuda.empty_cache()


def _graph_with_producer(torch, api, h, B, H, x_src, r_src, x_buf, r_buf, out):
    """One graph: a kernel writes x and residual from the source buffers (an
    elementwise multiply by one, so a real kernel node, not a memcpy node),
    then the fused layer on the same stream, PDL chaining on.  Returns the
    graph and the tensors its nodes read besides the caller's: they must
    outlive every replay (freed, their memory would go back to the caching
    allocator and be handed to the next input copied in).  """
    one = torch.ones((), dtype=torch.bfloat16, device="cuda")
    pad = torch.zeros(16 * 1024 * 1024, dtype=torch.float32, device="cuda")
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        # warm the elementwise kernels once outside capture
        pad.add_(1.0)
        torch.mul(x_src, one, out=x_buf)
        torch.mul(r_src, one, out=r_buf)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            pad.add_(1.0)                          # a longer kernel ahead of the producers
            torch.mul(r_src, one, out=r_buf)
            torch.mul(x_src, one, out=x_buf)       # the layer's direct predecessor
            api.moe_layer_forward(h, None, x_buf, r_buf, out, B, stream=torch.cuda.current_stream())
    return g, (one, pad)


@pytest.mark.parametrize("which,B,reps", [("tiny", 1, 12), ("tiny", 33, 6), ("full", 1, 6)])
def test_inputs_written_on_stream_before_the_layer(torch_cuda, which, B, reps):
    from sparse_moe_decode_router_b200 import api
    torch = torch_cuda
    if which == "tiny":
        base = synth.CONFIGS[0]
        dl = make_device_layer(base.with_(hidden=512, inter=256, shared_inter=64) if B > 8 else base)
    else:
        dl = make_device_layer(synth.CONFIGS[1])
    c = dl.cfg
    H, k, E = c.hidden, c.top_k, c.n_experts
    h = create_layer(dl, B)
    try:
        x_src = torch.empty((B, H), dtype=torch.bfloat16, device="cuda")
        r_src = torch.empty_like(x_src)
        x_buf = torch.empty_like(x_src)
        r_buf = torch.empty_like(x_src)
        out = torch.empty_like(x_src)
        g, keep = _graph_with_producer(torch, api, h, B, H, x_src, r_src, x_buf, r_buf, out)
        outs, plans, xs, rs, xbufs = [], [], [], [], []
        for rep in range(reps):
            ids = list(range(1000 + rep * B, 1000 + (rep + 1) * B))
            x_h, x_d = dl.tokens(ids)
            r_h, r_d = residual_tokens(c, ids)
            x_src.copy_(x_d)
            r_src.copy_(r_d)
            g.replay()
            outs.append(out.clone())
            torch.cuda.synchronize()
            plans.append(layer_routing_host(h, B, k, E))
            xbufs.append(to_host_u16(x_buf))
            xs.append(x_h)
            rs.append(r_h)
        assert api.moe_layer_last_device_error(h) == api.MOE_OK
        del g, keep
    finally:
        api.moe_layer_destroy(h)
    bad = []
    for rep in range(reps):
        assert np.array_equal(xbufs[rep], xs[rep]), f"replay {rep}: the producer did not write x"
        ref = oracle_layer_for(dl, xs[rep], rs[rep])
        try:
            assert_routing_equal(plans[rep], ref, W_ABS)
            ok, info = bf16_close(to_host_u16(outs[rep]), ref["out_bf16"])
            assert ok, info
        except AssertionError as e:
            prev = oracle.routing(xs[rep - 1], dl.router_w_host, dl.bias_host, k)["topk_idx"] if rep else None
            bad.append((rep, str(e)[:80], plans[rep]["topk_idx"].tolist(), ref["topk_idx"].tolist(),
                        None if prev is None else prev.tolist()))
    assert not bad, bad
