"""The routed-expert tolerance in helpers.py is derived from the GPU's rounding
points, not fitted to GPU results.  This CPU test re-derives it: it applies
exactly those roundings (f16 activations scaled by a power of two, f16 products
and eight-term f16 partial sums per 32-element block, fp32 across blocks, h
rounded to f16 before the down projection) in numpy to one expert of a
medium-size layer, and checks the resulting error against the fp64 oracle.
It uses no GPU code; the oracle supplies the reference."""
import numpy as np

import oracle
import synth
from helpers import OUT_MAX_REL, OUT_MEAN_REL, Y_ROUTED_MAX_REL, Y_ROUTED_MEAN_REL, metric_close

_E2M1 = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -0., -.5, -1, -1.5, -2, -3, -4, -6])


def _stage_f16(v):
    """f16 copy of a vector with max|v| placed in [2^8, 2^9), and its exponent."""
    amax = float(np.abs(v).max())
    e = int(np.floor(np.log2(amax))) - 8 if amax > 0 else 0
    return (v * 2.0 ** -e).astype(np.float16).astype(np.float64), e


def _gemv_f16_blocks(codes, scales, xs, e):
    """Rows of MXFP4 times the staged vector: per 32-element block, two f16
    accumulators (even / odd element pairs), each half summing eight products
    with one rounding per multiply-add; the four partial sums in fp32; the
    block's E8M0 scale; fp32 across blocks."""
    R, K = codes.shape[0], xs.shape[0]
    w = np.empty((R, K))
    w[:, 0::2] = _E2M1[codes & 15]
    w[:, 1::2] = _E2M1[codes >> 4]
    prod = (w.reshape(R, K // 32, 32) * xs.reshape(K // 32, 32)[None]).astype(np.float64)
    tot = np.zeros(prod.shape[:2])
    for acc in range(2):            # accumulator: pairs j with j % 2 == acc
        for half in range(2):       # low / high element of the pair
            s = np.zeros(prod.shape[:2], dtype=np.float16)
            for j in range(acc, 16, 2):
                s = (prod[..., 2 * j + half] + s.astype(np.float64)).astype(np.float16)
            tot += s.astype(np.float32).astype(np.float64)
    sc = 2.0 ** (scales.astype(np.float64) - 127)
    return (tot * sc).astype(np.float32).astype(np.float64).sum(1) * 2.0 ** e


def test_f16_block_partial_sums_fit_the_stated_bounds():
    cfg = synth.CONFIGS[0].with_(hidden=2048, inter=1024, shared_inter=0, n_experts=8, top_k=2,
                                 seed=synth.CONFIGS[0].seed + 900)
    wr = synth.gen_router_w(cfg)
    x_bf, _ = synth.gen_tokens(cfg, wr, None, [0])
    x = synth.bf16_to_f32(x_bf[0]).astype(np.float64)
    I = cfg.inter
    ys_gpu, ys_ref = [], []
    for expert in range(2):
        gc, gs, dc, ds = synth.gen_expert(cfg, expert)
        _, y_ref = oracle.expert_ffn(x, gc, gs, dc, ds)
        xs, ex = _stage_f16(x)
        gu = _gemv_f16_blocks(gc, gs, xs, ex)
        g, u = gu[:I], gu[I:]
        h = g / (1 + np.exp(-g)) * u
        hs, eh = _stage_f16(h)
        ys_gpu.append(_gemv_f16_blocks(dc, ds, hs, eh))
        ys_ref.append(y_ref)
    yg, yr = np.stack(ys_gpu), np.stack(ys_ref)
    ok, info = metric_close(yg, yr, Y_ROUTED_MAX_REL, Y_ROUTED_MEAN_REL)
    assert ok, info
    # the bounds keep a margin over what these roundings produce
    assert info["mean_rel"] < Y_ROUTED_MEAN_REL / 2, info
    assert info["max_abs"] < Y_ROUTED_MAX_REL / 2 * info["max_ref"], info
    # and the routed part of a layer output built from them stays far inside
    # the stated output tolerance (residual 0: the strictest case)
    w = np.array([0.6, 0.4])
    out_g = synth.bf16_to_f32(synth.bf16_rne((w @ yg).astype(np.float32))).astype(np.float64)
    out_r = synth.bf16_to_f32(synth.bf16_rne((w @ yr).astype(np.float32))).astype(np.float64)
    ok, info = metric_close(out_g, out_r, OUT_MAX_REL, OUT_MEAN_REL)
    assert ok, info
