"""CPU checks of the seeded input generator (synth): Philox known answers,
the Irwin-Hall draw, bf16 rounding, the MXFP4 quantiser and the routing-gap
conditioning, and the exact-tie router inputs.  The device generator's
bit-identity is checked in test_gpu_parity.py."""
import numpy as np
import pytest

import oracle
import synth
from helpers import TIE_SHAPES


def test_philox4x32_10_known_answers():
    # known-answer vectors of the Random123 distribution (Salmon et al., SC'11)
    kat = [
        ((0, 0, 0, 0), (0, 0), (0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8)),
        ((0xFFFFFFFF,) * 4, (0xFFFFFFFF, 0xFFFFFFFF), (0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD)),
        ((0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344), (0xA4093822, 0x299F31D0),
         (0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1)),
    ]
    for ctr, key, want in kat:
        got = synth.philox4x32_10(*ctr, *key)
        assert tuple(int(g) for g in got) == want


def test_irwin_hall_draw_moments_and_range():
    key = synth.stream_key(123, 0, synth.T_X)
    s = synth.irwin_hall_ints(key, 0, 0, 0, 400_000).astype(np.float64)
    assert s.min() >= -131070 and s.max() <= 131070
    assert abs(s.mean()) < 3 * synth.IH_SD / np.sqrt(len(s)) * 2
    assert abs(s.std() / synth.IH_SD - 1) < 0.01
    v = synth.normal_f32(key, 0, 0, 0, 400_000, 0.02).astype(np.float64)
    assert abs(v.std() / 0.02 - 1) < 0.01
    # substreams differ, elements are reproducible one by one
    a = synth.irwin_hall_ints(key, 1, 0, 100, 10)
    b = np.array([synth.irwin_hall_ints(key, 1, 0, 100 + i, 1)[0] for i in range(10)])
    assert np.array_equal(a, b)
    assert not np.array_equal(a, synth.irwin_hall_ints(key, 2, 0, 100, 10))


def test_bf16_rne_matches_torch():
    import torch
    rng = np.random.default_rng(2)
    v = np.concatenate([rng.normal(0, 1, 10000), rng.normal(0, 1e-30, 100)]).astype(np.float32)
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(synth.bf16_rne(v), want)
    assert np.array_equal(synth.bf16_to_f32(synth.bf16_rne(v)),
                          torch.from_numpy(v).to(torch.bfloat16).float().numpy())


def _dequant(codes, scales, K):
    return np.stack([oracle.dequant_row(codes[r], scales[r], K) for r in range(codes.shape[0])])


def test_quantizer_round_trips_exact_values_and_bounds_error():
    rng = np.random.default_rng(4)
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    R, K = 8, 128
    vals = mags[rng.integers(0, 8, (R, K))] * rng.choice([-1.0, 1.0], (R, K))
    vals *= np.repeat(2.0 ** rng.integers(-12, 3, (R, K // 32)), 32, axis=1)
    vals[:, :32] = 0.0                                   # an all-zero block
    codes, scales = synth.quantize_mxfp4(vals.astype(np.float32))
    assert np.array_equal(_dequant(codes, scales, K), vals)
    assert np.all(scales[:, 0] == 0)
    # arbitrary values: error at most one grid step of the block (2 * 2^(s-127))
    v = rng.normal(0, 0.02, (R, K)).astype(np.float32)
    codes, scales = synth.quantize_mxfp4(v)
    dq = _dequant(codes, scales, K)
    step = np.repeat(2.0 ** (scales.astype(np.float64) - 127) * 2, 32, axis=1)
    assert np.all(np.abs(dq - v) <= step)
    # the block maximum lands in the top binade [4, 6] of the grid
    amax_code = np.abs(dq).reshape(R, K // 32, 32).max(2) / 2.0 ** (scales.astype(np.float64) - 127)
    assert np.all((amax_code >= 4) & (amax_code <= 6))


def test_quantizer_ties_round_to_even():
    # scale 127 (amax 6 in the block): 0.25 -> 0, 0.75 -> 1, 1.25 -> 1, 1.75 -> 2, 2.5 -> 2, 3.5 -> 4, 5 -> 4
    row = np.zeros((1, 32), np.float32)
    row[0, :8] = [6, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5]
    codes, scales = synth.quantize_mxfp4(row)
    assert scales[0, 0] == 127
    dq = oracle.dequant_row(codes[0], scales[0], 32)
    assert list(dq[:8]) == [6, 0, 1, 1, 2, 2, 4, 4]


def test_tiny_workload_gap_and_bias():
    cfg = synth.CONFIGS[0]
    wr = synth.gen_router_w(cfg)
    x, att = synth.gen_tokens(cfg, wr, None, range(16))
    lg = oracle.router_logits(x, wr, None)
    srt = -np.sort(-lg, axis=1)
    assert np.all(srt[:, cfg.top_k - 1] - srt[:, cfg.top_k] >= cfg.min_gap)
    b = synth.gen_router_bias(synth.CONFIGS[3])
    ranks = np.rint(np.exp(-b.astype(np.float64) / 1.1)).astype(int)
    assert sorted(ranks.tolist()) == list(range(1, 897))
    assert synth.gen_router_bias(cfg) is None


def test_counted_bytes_formula():
    c1 = synth.CONFIGS[1]
    # per active expert: codes + scales of gate/up and down
    assert c1.expert_bytes() == 2 * 2048 * (3584 + 224) + 7168 * (1024 + 64)
    assert c1.counted_bytes(16) == 16 * c1.expert_bytes() + 3 * 2048 * 7168 * 2 + 7168 * 896 * 2 + 3 * 7168 * 2


@pytest.mark.parametrize("E,k,copies", TIE_SHAPES)
@pytest.mark.parametrize("with_bias", [True, False])
def test_tied_router_inputs_tie_at_the_selection_boundary(E, k, copies, with_bias):
    """The premise of the GPU tie test: every logit is an integer (so fp32
    and fp64 agree exactly), the copies of a group share every logit, and
    among the first tokens some have equal k-th and (k+1)-th logits, so
    their selected set depends on the tie rule."""
    cfg = synth.CONFIGS[0].with_(n_experts=E, top_k=k)
    wr, bias, group = synth.gen_tied_router(cfg, n_copies=copies, with_bias=with_bias)
    assert np.bincount(group).tolist() == [copies] * (E // copies)
    x = synth.gen_tied_tokens(cfg, 64)
    assert set(np.unique(synth.bf16_to_f32(x))) <= {-1.0, 0.0, 1.0}
    assert not np.any(synth.bf16_to_f32(x[0]))
    lg = synth.bf16_to_f32(x).astype(np.float64) @ synth.bf16_to_f32(wr).astype(np.float64)
    if bias is not None:
        lg += bias
    assert np.array_equal(lg, np.rint(lg)) and np.abs(lg).max() < 2.0 ** 24
    for g in range(E // copies):      # copies of a group tie on every token
        cols = lg[:, group == g]
        assert np.all(cols == cols[:, :1])
    srt = -np.sort(-lg, axis=1)
    boundary = srt[:, k - 1] == srt[:, k]
    assert boundary[:7].any() and boundary.sum() >= 4


def test_verify_positions_share_their_sequence_draw():
    """Verify-shape batches: the 8 positions of one sequence mix the
    sequence's draw (weight sqrt(0.9)) with their own, so they are strongly
    correlated with each other and route to far fewer distinct experts than
    independent tokens; positions of different sequences are independent."""
    cfg = synth.CONFIGS[5].with_(hidden=1024, n_experts=256)
    wr = synth.gen_router_w(cfg)
    x, _ = synth.gen_tokens(cfg, wr, None, range(16))
    xf = synth.bf16_to_f32(x).astype(np.float64)
    c = np.corrcoef(xf)
    within = c[:8, :8][~np.eye(8, dtype=bool)]
    across = c[:8, 8:]
    assert within.min() > 0.8 and np.abs(across).max() < 0.2
    ind = synth.CONFIGS[2].with_(hidden=1024, n_experts=256)
    xi, _ = synth.gen_tokens(ind, synth.gen_router_w(ind), None, range(8))
    lg_v = xf[:8] @ synth.bf16_to_f32(wr).astype(np.float64)
    lg_i = synth.bf16_to_f32(xi).astype(np.float64) @ synth.bf16_to_f32(synth.gen_router_w(ind)).astype(np.float64)
    top = lambda lg: len(np.unique(np.argsort(-lg, axis=1)[:, :16]))
    assert top(lg_v) < 0.6 * top(lg_i)


def test_edge_mxfp4_generator_covers_the_format():
    cfg = synth.CONFIGS[0]
    codes, scales = synth.gen_edge_mxfp4(cfg, 3, 8, 128, synth.T_EXPERT_GU, 87, 139)
    nib = np.stack([codes & 15, codes >> 4], -1).reshape(-1, 32)
    assert all((np.bincount(b, minlength=16) == 2).all() for b in nib)   # every code twice per block
    s = scales.reshape(-1)
    assert (s == 0).sum() == len(s[::23]) and s[s > 0].min() >= 87 and s.max() <= 139
    again = synth.gen_edge_mxfp4(cfg, 3, 8, 128, synth.T_EXPERT_GU, 87, 139)
    assert np.array_equal(again[0], codes) and np.array_equal(again[1], scales)   # seeded
    other = synth.gen_edge_mxfp4(cfg, 3, 8, 128, synth.T_EXPERT_D, 87, 139)
    assert not np.array_equal(other[0], codes)


def test_wide_range_tokens_keep_the_routing_margin():
    cfg = synth.CONFIGS[0]
    wr = synth.gen_router_w(cfg)
    x, _ = synth.gen_tokens(cfg, wr, None, range(6), tiny_every=7)
    xf = np.abs(synth.bf16_to_f32(x).astype(np.float64))
    ratio = xf[:, ::7].max(axis=1) / xf.max(axis=1)
    assert (ratio < 2.0 ** -26).all()                       # elements ~2^30 below the row's maximum
    for row in x:
        lg = synth.bf16_to_f32(row).astype(np.float64) @ synth.bf16_to_f32(wr).astype(np.float64)
        srt = np.sort(lg)[::-1]
        assert srt[cfg.top_k - 1] - srt[cfg.top_k] >= cfg.min_gap


_FULL_ROUTER = {}


def _full_router_w(cfg):
    """The full-size router matrix (the same draw for every full-size workload
    of one seed), generated once per test session."""
    key = (cfg.seed, cfg.hidden, cfg.n_experts, cfg.router_sigma)
    if key not in _FULL_ROUTER:
        _FULL_ROUTER[key] = synth.gen_router_w(cfg)
    return _FULL_ROUTER[key]


@pytest.mark.parametrize("cfg_id", [1, 2, 3, 5])
def test_full_size_bench_tokens_keep_the_routing_margin(cfg_id):
    """The first batch the bench times on each full-size workload (token ids
    0 .. B-1): the C++ oracle's fp64 logits, Zipf bias included, leave at least
    min_gap between the k-th and (k+1)-th score, so the expert set the GPU
    parity tests compare bit for bit is unique; the oracle's selection is
    exactly the experts above that boundary.  The generator measures the gap
    with its own numpy product, so this pins the two against each other at
    full size."""
    cfg = synth.CONFIGS[cfg_id]
    wr = _full_router_w(cfg)
    bias = synth.gen_router_bias(cfg)
    x, _ = synth.gen_tokens(cfg, wr, bias, range(cfg.batch))
    lg = oracle.router_logits(x, wr, bias)
    assert lg.shape == (cfg.batch, cfg.n_experts)
    srt = -np.sort(-lg, axis=1)
    k = cfg.top_k
    assert np.all(srt[:, k - 1] - srt[:, k] >= cfg.min_gap)
    rt = oracle.routing(x, wr, bias, k)
    for b in range(cfg.batch):
        above = np.flatnonzero(lg[b] >= srt[b, k - 1])
        assert np.array_equal(np.sort(rt["topk_idx"][b]), above)
    if cfg.verify_corr > 0:
        # positions of one sequence share experts (a verify step's routing)
        assert np.unique(rt["topk_idx"]).size < 0.75 * cfg.batch * k


def test_stack_workload_tokens_keep_the_routing_margin_on_every_layer():
    """The four-layer graph workload: each layer has its own router draw and
    its own token substream (token id = decode step); every (layer, step)
    token routes with the margin under the oracle's logits, and the layers'
    routers are different draws."""
    cfg = synth.CONFIGS[4]
    k = cfg.top_k
    first = None
    for layer in range(cfg.n_layers):
        wr = synth.gen_router_w(cfg, layer)
        if first is None:
            first = wr
        else:
            assert not np.array_equal(wr, first)
        x, _ = synth.gen_tokens(cfg, wr, None, range(cfg.n_steps), layer=layer)
        lg = oracle.router_logits(x, wr, None)
        srt = -np.sort(-lg, axis=1)
        assert np.all(srt[:, k - 1] - srt[:, k] >= cfg.min_gap)
