"""Pins for the oracle: each check ties an oracle function to something other
than itself (a hand-written table, brute force, a closed form, an invariant,
or a special case that reduces to a dense textbook computation).  CPU only."""
import itertools
import math
import os

import numpy as np
import pytest

import oracle
from synth import bf16_rne, bf16_to_f32

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

# exactly representable E2M1 magnitudes -> magnitude index (OCP MX v1.0 FP4 E2M1)
_MAG_INDEX = {0.0: 0, 0.5: 1, 1.0: 2, 1.5: 3, 2.0: 4, 3.0: 5, 4.0: 6, 6.0: 7}


def encode_exact(W, s=127):
    """Pack a matrix whose entries are exactly E2M1 * 2^(s-127) (one scale for
    every block) into codes [R][K/2] + scales [R][K/32].  Test-side encoder."""
    W = np.asarray(W, dtype=np.float64)
    R, K = W.shape
    scale = 2.0 ** (s - 127)
    codes = np.zeros((R, K), dtype=np.uint8)
    for r in range(R):
        for c in range(K):
            v = W[r, c] / scale
            codes[r, c] = _MAG_INDEX[abs(v)] | (8 if v < 0 else 0)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return packed, np.full((R, K // 32), s, dtype=np.uint8)


def random_exact(rng, shape, s_choices=(124, 125, 126, 127)):
    """Random matrix on the E2M1 grid with a per-32-block random scale;
    returns (dense values, codes, scales)."""
    R, K = shape
    mags = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    idx = rng.integers(0, 8, size=(R, K))
    sign = rng.integers(0, 2, size=(R, K))
    s = rng.choice(np.array(s_choices), size=(R, K // 32))
    vals = mags[idx] * np.where(sign == 1, -1.0, 1.0) * np.repeat(2.0 ** (s - 127.0), 32, axis=1)
    codes = (idx | (sign << 3)).astype(np.uint8)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return vals, packed, s.astype(np.uint8)


def silu_np(g):
    return g / (1.0 + np.exp(-g))


# ---------------------------------------------------------------- dequant ---
def test_e2m1_e8m0_table_matches_hand_written_values():
    rows = []
    with open(os.path.join(GOLDEN, "e2m1_e8m0_table.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                c, s, v = line.split()
                rows.append((int(c), int(s), float(v)))
    assert len(rows) >= 60
    for code, s, v in rows:
        got = oracle.e2m1_value(code) * oracle.e8m0_value(s)
        if math.isnan(v):
            assert math.isnan(got)
        else:
            assert got == v, (code, s, got, v)
            assert math.copysign(1.0, got) == math.copysign(1.0, v) or v == 0


def test_dequant_row_nibble_order_and_scale_index():
    # byte 0x7A: low nibble 0xA (-1.0) is element 0, high nibble 0x7 (6.0) is element 1
    codes = np.zeros(32, dtype=np.uint8)
    codes[0] = 0x7A
    codes[16] = 0x3D          # element 32 = code 0xD (-3), element 33 = code 0x3 (1.5)
    scales = np.array([127, 128], dtype=np.uint8)   # second block doubled
    row = oracle.dequant_row(codes, scales, 64)
    assert row[0] == -1.0 and row[1] == 6.0
    assert row[32] == -6.0 and row[33] == 3.0
    assert np.all(row[2:32] == 0) and np.all(row[34:] == 0)


# ----------------------------------------------------------------- router ---
def test_router_logits_exact_on_integer_inputs():
    rng = np.random.default_rng(1)
    B, H, E = 3, 64, 12
    xi = rng.integers(-8, 9, size=(B, H))
    wi = rng.integers(-8, 9, size=(H, E))
    bias = rng.integers(-4, 5, size=E).astype(np.float32)
    x = bf16_rne(xi.astype(np.float32))
    wr = bf16_rne(wi.astype(np.float32))
    got = oracle.router_logits(x, wr, bias)
    want = (xi @ wi + bias.astype(np.int64)).astype(np.float64)   # exact integers
    assert np.array_equal(got, want)


def test_router_logits_transposition_pin():
    # one nonzero weight: logits[b][e] = x[b][h0] * w  only at e = e0
    B, H, E = 2, 32, 5
    x = np.zeros((B, H), np.float32)
    x[0, 3], x[1, 3] = 2.0, -0.5
    w = np.zeros((H, E), np.float32)
    w[3, 4] = 1.5
    got = oracle.router_logits(bf16_rne(x), bf16_rne(w))
    want = np.zeros((B, E))
    want[0, 4], want[1, 4] = 3.0, -0.75
    assert np.array_equal(got, want)


# ------------------------------------------------------------------ top-k ---
def brute_topk(lg, k):
    """All k-subsets; keep those with the largest sum; among them the
    lexicographically smallest ascending id tuple (lower id wins ties)."""
    best, best_sum = None, None
    for sub in itertools.combinations(range(len(lg)), k):
        s = sum(lg[i] for i in sub)
        if best is None or s > best_sum or (s == best_sum and sub < best):
            best, best_sum = sub, s
    return list(best)


@pytest.mark.parametrize("E,k", [(8, 1), (9, 3), (10, 4), (12, 2), (12, 5)])
def test_topk_matches_brute_force_with_ties(E, k):
    rng = np.random.default_rng(E * 31 + k)
    for _ in range(40):
        lg = rng.integers(-3, 4, size=(1, E)).astype(np.float64)   # many exact ties
        idx, w = oracle.topk_softmax(lg, k)
        assert list(idx[0]) == brute_topk(list(lg[0]), k)


def test_topk_tiny_config_all_subsets():
    # the tiny workload's shape: 32 experts, top-4, all C(32,4) = 35960 subsets
    rng = np.random.default_rng(7)
    lg = rng.integers(-5, 6, size=(1, 32)).astype(np.float64)
    idx, _ = oracle.topk_softmax(lg, 4)
    assert list(idx[0]) == brute_topk(list(lg[0]), 4)


def test_softmax_closed_forms():
    # two selected logits: w = 1 / (1 + e^(l_other - l_self))
    lg = np.array([[0.3, 2.0, -1.0, 1.25]])
    idx, w = oracle.topk_softmax(lg, 2)
    assert list(idx[0]) == [1, 3]
    assert abs(w[0, 0] - 1.0 / (1.0 + math.exp(1.25 - 2.0))) < 1e-15
    assert abs(w[0, 1] - 1.0 / (1.0 + math.exp(2.0 - 1.25))) < 1e-15
    # k = 1: the weight is exactly one
    idx1, w1 = oracle.topk_softmax(lg, 1)
    assert idx1[0, 0] == 1 and w1[0, 0] == 1.0
    # equal selected logits: uniform weights
    idx4, w4 = oracle.topk_softmax(np.array([[5.0, 5.0, 5.0, 5.0, 1.0]]), 4)
    assert list(idx4[0]) == [0, 1, 2, 3] and np.all(w4 == 0.25)
    # weights sum to one and follow the logits' order
    rng = np.random.default_rng(3)
    lg = rng.normal(0, 4, size=(16, 40))
    idx, w = oracle.topk_softmax(lg, 7)
    assert np.all(np.abs(w.sum(1) - 1.0) < 1e-12)
    for b in range(16):
        sel = lg[b, idx[b]]
        assert np.all(np.diff(idx[b]) > 0)
        order = np.argsort(sel)
        assert np.all(np.diff(w[b, order]) >= 0)


# ---------------------------------------------------------------- buckets ---
def test_bucket_invariants():
    rng = np.random.default_rng(11)
    for B, k, E in [(1, 4, 32), (8, 16, 896), (64, 16, 896), (5, 3, 7)]:
        idx = np.stack([np.sort(rng.choice(E, size=k, replace=False)) for _ in range(B)]).astype(np.int32)
        r = oracle.bucket(idx, E)
        counts, offsets, pairs = r["counts"], r["offsets"], r["pair_ids"]
        assert counts.sum() == B * k
        assert offsets[0] == 0 and offsets[E] == B * k
        assert np.array_equal(np.diff(offsets), counts)
        assert np.array_equal(np.sort(pairs), np.arange(B * k))          # a permutation
        flat = idx.reshape(-1)
        for e in range(E):
            seg = pairs[offsets[e]:offsets[e + 1]]
            assert np.all(flat[seg] == e)                                 # bucket holds its expert
            assert np.all(np.diff(seg) > 0)                               # stable: (b, j) order
        assert np.array_equal(r["active"], np.nonzero(counts)[0])
        assert r["n_active"] == np.count_nonzero(counts)


# ------------------------------------------------------------------ SwiGLU --
def test_silu_closed_forms():
    assert oracle.silu(0.0) == 0.0
    assert abs(oracle.silu(math.log(3.0)) - 0.75 * math.log(3.0)) < 1e-15   # sigmoid(ln 3) = 3/4
    for g in (0.1, 1.0, 2.5, 7.0):
        assert abs(oracle.silu(-g) - (oracle.silu(g) - g)) < 1e-14         # silu(-g) = silu(g) - g
    assert abs(oracle.silu(40.0) - 40.0) < 1e-12


def test_expert_ffn_equals_dense_ffn_on_exact_weights():
    rng = np.random.default_rng(5)
    H, I = 96, 64
    Wgu, gc, gs = random_exact(rng, (2 * I, H))
    Wd, dc, ds = random_exact(rng, (H, I))
    x = rng.normal(0, 1, size=H)
    h, y = oracle.expert_ffn(x, gc, gs, dc, ds)
    g = Wgu[:I] @ x
    u = Wgu[I:] @ x
    h_ref = silu_np(g) * u
    y_ref = Wd @ h_ref
    assert np.allclose(h, h_ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(y, y_ref, rtol=1e-12, atol=1e-12)
    # swapping the gate and up halves changes the result (gate rows come first)
    h_sw = silu_np(u) * g
    assert not np.allclose(h, h_sw)


def test_shared_ffn_equals_dense_ffn():
    rng = np.random.default_rng(6)
    H, Is = 64, 32
    gu = bf16_rne(rng.normal(0, 0.1, size=(2 * Is, H)).astype(np.float32))
    d = bf16_rne(rng.normal(0, 0.1, size=(H, Is)).astype(np.float32))
    x = rng.normal(0, 1, size=H)
    h, y = oracle.shared_ffn(x, gu, d)
    G = bf16_to_f32(gu).astype(np.float64)
    D = bf16_to_f32(d).astype(np.float64)
    h_ref = silu_np(G[:Is] @ x) * (G[Is:] @ x)
    assert np.allclose(h, h_ref, rtol=1e-12, atol=1e-13)
    assert np.allclose(y, D @ h_ref, rtol=1e-12, atol=1e-13)


# ------------------------------------------------------------- bf16 round --
def test_round_bf16_against_fp32_path_and_ties():
    import torch
    rng = np.random.default_rng(9)
    v = np.concatenate([rng.normal(0, 1, 4000), rng.normal(0, 1e-3, 1000), rng.normal(0, 300, 1000)])
    v = v.astype(np.float32)     # fp32-representable: one rounding either way
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.round_bf16(float(t)) for t in v], dtype=np.uint16)
    assert np.array_equal(got, want)
    # exact ties go to the even mantissa
    assert oracle.round_bf16(1.0 + 2 ** -8) == 0x3F80
    assert oracle.round_bf16(1.0 + 3 * 2 ** -8) == 0x3F82
    assert oracle.round_bf16(-(1.0 + 2 ** -8)) == 0xBF80
    # straight from double: no double rounding through fp32
    assert oracle.round_bf16(1.0 + 2 ** -8 + 2 ** -40) == 0x3F81
    assert oracle.round_bf16(0.0) == 0 and oracle.round_bf16(-0.0) == 0x8000


# ------------------------------------------------------------ whole layer --
def _tiny_layer_arrays(rng, B, H, E, k, I, Is, bias=False):
    wr = bf16_rne(rng.normal(0, 0.2, size=(H, E)).astype(np.float32))
    gu_vals, gc, gs = [], [], []
    d_vals, dc, ds = [], [], []
    for _ in range(E):
        a, b_, c = random_exact(rng, (2 * I, H), s_choices=(120, 121, 122))
        gu_vals.append(a), gc.append(b_), gs.append(c)
        a, b_, c = random_exact(rng, (H, I), s_choices=(120, 121, 122))
        d_vals.append(a), dc.append(b_), ds.append(c)
    sgu = bf16_rne(rng.normal(0, 0.05, size=(2 * Is, H)).astype(np.float32))
    sd = bf16_rne(rng.normal(0, 0.05, size=(H, Is)).astype(np.float32))
    x = bf16_rne(rng.normal(0, 1, size=(B, H)).astype(np.float32))
    res = bf16_rne(rng.normal(0, 1, size=(B, H)).astype(np.float32))
    bvec = rng.normal(0, 1, size=E).astype(np.float32) if bias else None
    return dict(wr=wr, gu_vals=np.stack(gu_vals), gc=np.stack(gc), gs=np.stack(gs),
                d_vals=np.stack(d_vals), dc=np.stack(dc), ds=np.stack(ds), sgu=sgu, sd=sd,
                x=x, res=res, bias=bvec)


def _run(a, k, **kw):
    return oracle.layer(a["x"], a["res"], a["wr"], a["bias"], a["gc"], a["gs"], a["dc"], a["ds"],
                        a["sgu"], a["sd"], k, **kw)


def test_layer_equals_dense_moe_over_all_experts():
    """Evaluate every expert densely on every token and weight by the
    softmax over the selected logits (zero elsewhere): the sparse layer
    must agree with this dense formulation."""
    rng = np.random.default_rng(21)
    B, H, E, k, I, Is = 3, 64, 6, 2, 32, 32
    a = _tiny_layer_arrays(rng, B, H, E, k, I, Is, bias=True)
    r = _run(a, k)
    X = bf16_to_f32(a["x"]).astype(np.float64)
    Wr = bf16_to_f32(a["wr"]).astype(np.float64)
    lg = X @ Wr + a["bias"].astype(np.float64)
    G = bf16_to_f32(a["sgu"]).astype(np.float64)
    D = bf16_to_f32(a["sd"]).astype(np.float64)
    for b in range(B):
        sel = np.argsort(-lg[b], kind="stable")[:k]
        gate = np.zeros(E)
        z = np.exp(lg[b, sel] - lg[b, sel].max())
        gate[sel] = z / z.sum()
        acc = bf16_to_f32(a["res"][b]).astype(np.float64)
        acc = acc + D @ (silu_np(G[:Is] @ X[b]) * (G[Is:] @ X[b]))
        for e in range(E):
            Wgu, Wd = a["gu_vals"][e], a["d_vals"][e]
            acc = acc + gate[e] * (Wd @ (silu_np(Wgu[:I] @ X[b]) * (Wgu[I:] @ X[b])))
        assert np.allclose(r["out"][b], acc, rtol=1e-11, atol=1e-11)
        assert sorted(sel.tolist()) == list(r["topk_idx"][b])


def test_layer_hand_worked_example():
    """H = I = Is = 32, E = 4, k = 2, x = 2 e_0, residual = 0.25 everywhere.
    Router row 0 = [1, 0.5, -1, 0.25] -> logits [2, 1, -2, 0.5] -> experts
    {0, 1} with weights sigma(1), sigma(-1).  Expert 0: g_0 = 2, u_0 = 3,
    y_0 = 0.5 h_0.  Expert 1: g_0 = -2, u_0 = 2, y_1 = 2 h_0.  Shared:
    g_0 = 1, u_0 = 2, y_2 = h_0.  Every other weight is zero."""
    H = I = Is = 32
    E, k = 4, 2
    x = np.zeros((1, H), np.float32)
    x[0, 0] = 2.0
    res = np.full((1, H), 0.25, np.float32)
    wr = np.zeros((H, E), np.float32)
    wr[0] = [1.0, 0.5, -1.0, 0.25]
    gu = np.zeros((E, 2 * I, H))
    dn = np.zeros((E, H, I))
    gu[0, 0, 0], gu[0, I + 0, 0], dn[0, 0, 0] = 1.0, 1.5, 0.5
    gu[1, 0, 0], gu[1, I + 0, 0], dn[1, 1, 0] = -1.0, 1.0, 2.0
    enc = [encode_exact(gu[e]) for e in range(E)]
    encd = [encode_exact(dn[e]) for e in range(E)]
    sgu = np.zeros((2 * Is, H), np.float32)
    sd = np.zeros((H, Is), np.float32)
    sgu[0, 0], sgu[Is, 0], sd[2, 0] = 0.5, 1.0, 1.0
    r = oracle.layer(bf16_rne(x), bf16_rne(res), bf16_rne(wr), None,
                     np.stack([c for c, _ in enc]), np.stack([s for _, s in enc]),
                     np.stack([c for c, _ in encd]), np.stack([s for _, s in encd]),
                     bf16_rne(sgu), bf16_rne(sd), k)
    sig = lambda t: 1.0 / (1.0 + math.exp(-t))
    w0, w1 = sig(1.0), sig(-1.0)
    assert list(r["topk_idx"][0]) == [0, 1]
    assert abs(r["topk_w"][0, 0] - w0) < 1e-15 and abs(r["topk_w"][0, 1] - w1) < 1e-15
    want = np.full(H, 0.25)
    want[0] += w0 * 0.5 * (2.0 * sig(2.0)) * 3.0
    want[1] += w1 * 2.0 * (-2.0 * sig(-2.0)) * 2.0
    want[2] += (1.0 * sig(1.0)) * 2.0
    assert np.allclose(r["out"][0], want, rtol=0, atol=1e-14)
    assert r["n_active"] == 2 and list(r["active"]) == [0, 1]
    assert list(r["offsets"][:5]) == [0, 1, 2, 2, 2]


def test_layer_special_cases():
    rng = np.random.default_rng(33)
    B, H, E, k, I, Is = 4, 64, 8, 3, 32, 32
    a = _tiny_layer_arrays(rng, B, H, E, k, I, Is)
    base = _run(a, k)
    # (a) zero experts and zero shared expert: out = bf16(residual)
    z = dict(a, gc=np.zeros_like(a["gc"]), dc=np.zeros_like(a["dc"]),
             sgu=np.zeros_like(a["sgu"]), sd=np.zeros_like(a["sd"]))
    rz = _run(z, k)
    assert np.array_equal(rz["out_bf16"], a["res"])
    # (b) k = 1, zero shared, zero residual: out = bf16(FFN_e(x)) with e the argmax
    one = dict(a, sgu=np.zeros_like(a["sgu"]), res=np.zeros_like(a["res"]))
    r1 = _run(one, 1)
    for b in range(B):
        e = int(r1["topk_idx"][b, 0])
        _, y = oracle.expert_ffn(bf16_to_f32(a["x"][b]).astype(np.float64), a["gc"][e], a["gs"][e],
                                 a["dc"][e], a["ds"][e])
        assert np.array_equal(r1["out"][b], y)
        assert np.array_equal(r1["out_bf16"][b], np.array([oracle.round_bf16(t) for t in y], np.uint16))
    # (c) tokens are independent of the rest of the batch
    for b in range(B):
        rb = oracle.layer(a["x"][b:b + 1], a["res"][b:b + 1], a["wr"], None, a["gc"], a["gs"],
                          a["dc"], a["ds"], a["sgu"], a["sd"], k)
        assert np.array_equal(rb["out"][0], base["out"][b])
    # (d) relabelling experts (router columns and tensors together) changes nothing but ids
    perm = rng.permutation(E)              # new id of old expert e is perm[e]
    inv = np.argsort(perm)
    rl = dict(a, wr=a["wr"][:, inv], gc=a["gc"][inv], gs=a["gs"][inv], dc=a["dc"][inv], ds=a["ds"][inv])
    rp = _run(rl, k)
    assert np.allclose(rp["out"], base["out"], rtol=1e-12, atol=1e-12)
    for b in range(B):
        assert sorted(perm[base["topk_idx"][b]].tolist()) == list(rp["topk_idx"][b])
    # (e) raising every down-projection scale byte by one doubles the routed part exactly
    dbl = dict(a, ds=(a["ds"] + 1).astype(np.uint8))
    rd = _run(dbl, k)
    resid = bf16_to_f32(a["res"]).astype(np.float64)
    routed = base["out"] - resid - base["y_shared"]
    routed2 = rd["out"] - resid - rd["y_shared"]
    assert np.allclose(routed2, 2 * routed, rtol=1e-12, atol=1e-12)
    # expert-slot addressing: a compact copy of only the selected experts gives the same result
    sel = np.unique(base["topk_idx"])
    rc = oracle.layer(a["x"], a["res"], a["wr"], None, a["gc"][sel], a["gs"][sel], a["dc"][sel],
                      a["ds"][sel], a["sgu"], a["sd"], k, experts=sel)
    assert np.array_equal(rc["out"], base["out"])


# ------------------------------------------- router and shared variants ----
def test_sigmoid_topk_brute_force_with_bias_and_ties():
    """Sigmoid scoring: the selected set maximises sum(sigmoid(l) + bias) over
    all k-subsets (lower ids win ties), whatever the bias does to the order."""
    rng = np.random.default_rng(91)
    for E, k in ((8, 2), (10, 3), (12, 4)):
        for _ in range(30):
            lg = rng.integers(-3, 4, size=(1, E)).astype(np.float64)
            bias = (rng.integers(-2, 3, size=E) * 0.25).astype(np.float32)
            idx, w = oracle.topk_sigmoid(lg, k, bias)
            score = [1.0 / (1.0 + math.exp(-lg[0, e])) + float(bias[e]) for e in range(E)]
            assert list(idx[0]) == brute_topk(score, k)
            assert abs(w.sum() - 1.0) < 1e-12


def test_sigmoid_weights_closed_forms():
    # l = (0, ln 3): sigmoid = (1/2, 3/4) -> weights (2/5, 3/5)
    idx, w = oracle.topk_sigmoid(np.array([[0.0, math.log(3.0)]]), 2)
    assert list(idx[0]) == [0, 1]
    assert abs(w[0, 0] - 0.4) < 1e-15 and abs(w[0, 1] - 0.6) < 1e-15
    # the bias steers the choice but stays out of the weights: sigmoid(2.0) >
    # sigmoid(1.9), yet +0.1 on expert 1 selects it, alone, with weight 1
    idx, w = oracle.topk_sigmoid(np.array([[2.0, 1.9]]), 1, np.array([0.0, 0.1], np.float32))
    assert list(idx[0]) == [1] and w[0, 0] == 1.0
    # with k = 2 both are selected and the weights ignore the bias
    idx, w = oracle.topk_sigmoid(np.array([[2.0, 1.9]]), 2, np.array([0.0, 0.1], np.float32))
    s0, s1 = 1 / (1 + math.exp(-2.0)), 1 / (1 + math.exp(-1.9))
    assert abs(w[0, 0] - s0 / (s0 + s1)) < 1e-15 and abs(w[0, 1] - s1 / (s0 + s1)) < 1e-15


def test_sigmoid_without_bias_selects_like_softmax():
    # sigmoid is increasing: without a bias both scorings select the same set
    rng = np.random.default_rng(92)
    lg = rng.normal(0, 2, size=(16, 40))
    i1, _ = oracle.topk_sigmoid(lg, 6)
    i2, _ = oracle.topk_softmax(lg, 6)
    assert np.array_equal(i1, i2)


def test_layer_sigmoid_scoring_matches_dense_formulation():
    rng = np.random.default_rng(93)
    B, H, E, k, I, Is = 3, 64, 6, 2, 32, 32
    a = _tiny_layer_arrays(rng, B, H, E, k, I, Is, bias=True)
    r = _run(a, k, scoring="sigmoid")
    X = bf16_to_f32(a["x"]).astype(np.float64)
    Wr = bf16_to_f32(a["wr"]).astype(np.float64)
    lg = X @ Wr                                   # raw logits: the bias only steers
    assert np.allclose(r["logits"], lg, rtol=0, atol=1e-12)
    G = bf16_to_f32(a["sgu"]).astype(np.float64)
    D = bf16_to_f32(a["sd"]).astype(np.float64)
    for b in range(B):
        s = 1.0 / (1.0 + np.exp(-lg[b]))
        sel = sorted(brute_topk(list(s + a["bias"].astype(np.float64)), k))
        assert list(r["topk_idx"][b]) == sel
        acc = bf16_to_f32(a["res"][b]).astype(np.float64)
        acc = acc + D @ (silu_np(G[:Is] @ X[b]) * (G[Is:] @ X[b]))
        for e in sel:
            h = silu_np(a["gu_vals"][e][:I] @ X[b]) * (a["gu_vals"][e][I:] @ X[b])
            acc = acc + s[e] / s[sel].sum() * (a["d_vals"][e] @ h)
        assert np.allclose(r["out"][b], acc, rtol=1e-12, atol=1e-12)


def test_mxfp4_shared_expert_equals_bf16_copy_and_expert_ffn():
    """An MXFP4 shared expert whose values are exact in bf16 gives the bf16
    shared expert's result bit for bit, and equals the MXFP4 expert FFN."""
    rng = np.random.default_rng(94)
    B, H, E, k, I, Is = 2, 64, 4, 2, 32, 64
    a = _tiny_layer_arrays(rng, B, H, E, k, I, Is)
    gv, gc, gs = random_exact(rng, (2 * Is, H), s_choices=(119, 121, 123))
    dv, dc, ds = random_exact(rng, (H, Is), s_choices=(119, 121, 123))
    r_mx = _run(a, k, shared_mx=(gc, gs, dc, ds))
    r_bf = _run(dict(a, sgu=bf16_rne(gv.astype(np.float32)), sd=bf16_rne(dv.astype(np.float32))), k)
    assert np.array_equal(bf16_to_f32(bf16_rne(gv.astype(np.float32))).astype(np.float64), gv)
    assert np.array_equal(r_mx["y_shared"], r_bf["y_shared"])
    assert np.array_equal(r_mx["out"], r_bf["out"])
    for b in range(B):
        _, y = oracle.expert_ffn(bf16_to_f32(a["x"][b]).astype(np.float64), gc, gs, dc, ds)
        assert np.array_equal(r_mx["y_shared"][b], y)
