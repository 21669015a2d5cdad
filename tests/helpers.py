"""Shared test helpers: tolerance metrics and oracle runs on device workloads."""
import numpy as np

from synth import bf16_to_f32

# Layer output tolerance (bf16 [B][H]) stated for the layer:
#   max|out - ref| <= 1e-2 * max|ref|  and  sum|out - ref| / sum|ref| <= 2e-3,
# ref = the oracle's fp64 result rounded once to bf16.
OUT_MAX_REL = 1e-2
OUT_MEAN_REL = 2e-3
# fp32 intermediates against fp64.  Shared-expert output: bf16 weights times
# fp32 activations, fp32 sums (K <= 7168) -> relative error near 1e-6; the
# bounds leave an order of magnitude of margin.
Y_MAX_REL = 1e-4
Y_MEAN_REL = 1e-5
# Routed expert outputs.  MXFP4 dot products take their products and their
# partial sums over eight products in f16 (unit roundoff u = 2^-11 ~ 4.9e-4 per
# operation), the down projection reads the SwiGLU activations h rounded once
# to f16, and block sums are scaled and accumulated in fp32.  For the
# random-sign data here the errors do not line up: an exact emulation of these
# roundings on the full-size layer (one token, its 16 experts) gives a mean
# relative error of ~7.4e-4 and a max error of ~8.8e-4 * max|y|.  The bounds
# leave a factor of ~2.7 (mean) and ~4.5 (max) of margin; the layer output
# keeps its own, stated tolerance above.
Y_ROUTED_MAX_REL = 4e-3
Y_ROUTED_MEAN_REL = 2e-3
# routing weights: fp32 softmax of fp32 logits vs fp64 (|w| <= 1)
W_ABS = 1e-5

# Exact-tie router workloads (synth.gen_tied_router): (n_experts, top_k,
# copies per tied group).  They cover the top-k kernel's slice layouts: one,
# four and four candidates per lane in the first stage.
TIE_SHAPES = ((32, 4, 8), (896, 16, 4), (1024, 32, 4))


def bf16_close(gpu_u16, ref_u16, max_rel=OUT_MAX_REL, mean_rel=OUT_MEAN_REL):
    g = bf16_to_f32(np.asarray(gpu_u16)).astype(np.float64)
    r = bf16_to_f32(np.asarray(ref_u16)).astype(np.float64)
    return metric_close(g, r, max_rel, mean_rel)


def metric_close(g, r, max_rel, mean_rel):
    g = np.asarray(g, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.all(np.isfinite(g)), "non-finite values in GPU output"
    d = np.abs(g - r)
    mx, mr = d.max(), d.sum() / max(np.abs(r).sum(), 1e-300)
    ok = mx <= max_rel * np.abs(r).max() and mr <= mean_rel
    return ok, dict(max_abs=float(mx), max_ref=float(np.abs(r).max()), mean_rel=float(mr))
