"""Seeded synthetic inputs for the sparse MXFP4 MoE decode layer.

This module makes INPUTS only: weights, activations and the router bias of
the five workloads (tiny B=1; full-size B=1, B=8, B=64 with a Zipf-skewed
router; a 4-layer full-size stack).  It holds none of the layer's own
arithmetic (no dequantisation, no GEMV, no top-k, no SwiGLU).  It serves
both the oracle (tests) and the CUDA path (tests, bench) so that both see
bit-identical inputs.

Random numbers come from the counter-based generator Philox4x32-10
(Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as 1, 2, 3",
SC'11), so any element of any tensor can be regenerated on its own, on the
host (numpy, here) or on the device (synth_gen.cu), with the same bits.

Value recipe (all integer or single IEEE-754 fp32 operations, so host and
device agree bit for bit):

* a "normal" draw of standard deviation sigma is the Irwin-Hall sum of four
  16-bit uniforms, centred, as an exact fp32 integer S, times the fp32
  constant sigma/sd(S) in ONE fp32 multiply (round to nearest even);
  the tails are bounded at 3.46 sigma, mean and variance are exact;
* bf16 tensors are the fp32 draws rounded to nearest even;
* MXFP4 tensors quantise the fp32 draws per 32-element block along K:
  E8M0 scale byte s = floor(log2(amax)) - 2 + 127 (amax = 0 gives s = 0),
  then each value divided by 2^(s-127) (an exact power-of-two multiply) and
  rounded to nearest even onto the E2M1 grid {0, .5, 1, 1.5, 2, 3, 4, 6},
  saturating at 6; code = sign << 3 | magnitude index; two codes per byte,
  the even-K element in the low nibble.

The MXFP4 element and scale formats follow the OCP Microscaling Formats
(MX) v1.0 specification; the pages on the decode path only say the experts
use native MXFP4 4-bit weights (tmtpost page, section on the phenomenon).
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass, replace

import numpy as np

# --------------------------------------------------------------------------
# Philox4x32-10
# --------------------------------------------------------------------------
_MASK = np.uint64(0xFFFFFFFF)
_M0 = np.uint64(0xD2511F53)
_M1 = np.uint64(0xCD9E8D57)
_W0 = 0x9E3779B9
_W1 = 0xBB67AE85


def philox4x32_10(c0, c1, c2, c3, k0: int, k1: int):
    """Vectorised Philox4x32 with 10 rounds.  Counters are uint32 arrays
    (or scalars), the key is two uint32 scalars.  Returns four uint32 arrays."""
    c0 = np.asarray(c0, dtype=np.uint64)
    c1 = np.asarray(c1, dtype=np.uint64)
    c2 = np.asarray(c2, dtype=np.uint64)
    c3 = np.asarray(c3, dtype=np.uint64)
    c0, c1, c2, c3 = np.broadcast_arrays(c0, c1, c2, c3)
    ka, kb = int(k0) & 0xFFFFFFFF, int(k1) & 0xFFFFFFFF
    for r in range(10):
        if r:
            ka = (ka + _W0) & 0xFFFFFFFF
            kb = (kb + _W1) & 0xFFFFFFFF
        p0 = _M0 * c0
        p1 = _M1 * c2
        n0 = (p1 >> np.uint64(32)) ^ c1 ^ np.uint64(ka)
        n1 = p1 & _MASK
        n2 = (p0 >> np.uint64(32)) ^ c3 ^ np.uint64(kb)
        n3 = p0 & _MASK
        c0, c1, c2, c3 = n0, n1, n2, n3
    return (c0.astype(np.uint32), c1.astype(np.uint32),
            c2.astype(np.uint32), c3.astype(np.uint32))


# --------------------------------------------------------------------------
# Substreams
# --------------------------------------------------------------------------
T_ROUTER_W = 1
T_X = 2
T_RESIDUAL = 3
T_SHARED_GU = 4
T_SHARED_D = 5
T_EXPERT_GU = 6
T_EXPERT_D = 7
T_ZIPF_PERM = 8
T_TIES = 9
T_EDGE = 10
T_SHARED_MX_GU = 11
T_SHARED_MX_D = 12

# Irwin-Hall(4) of 16-bit uniforms: S = sum - 2*65535, Var(S) = 4*(65536^2-1)/12
IH_SD = math.sqrt(4.0 * (65536.0 * 65536.0 - 1.0) / 12.0)


def sigma_const(sigma: float) -> np.float32:
    """fp32 multiplier turning the integer Irwin-Hall sum into N(0, sigma^2)."""
    return np.float32(sigma / IH_SD)


def stream_key(seed: int, layer: int, tensor: int) -> tuple[int, int]:
    return seed & 0xFFFFFFFF, ((layer & 0xFFFF) << 16) | (tensor & 0xFFFF)


def irwin_hall_ints(key: tuple[int, int], sub0: int, sub1: int,
                    start: int, count: int) -> np.ndarray:
    """Centred integer Irwin-Hall sums for elements [start, start+count) of
    one substream.  Element n uses Philox counter (n>>1 lo, n>>1 hi, sub0,
    sub1) and output words (0,1) for even n, (2,3) for odd n."""
    n = np.arange(start, start + count, dtype=np.uint64)
    q = n >> np.uint64(1)
    o0, o1, o2, o3 = philox4x32_10(q & _MASK, q >> np.uint64(32),
                                   np.uint64(sub0 & 0xFFFFFFFF),
                                   np.uint64(sub1 & 0xFFFFFFFF), *key)
    odd = (n & np.uint64(1)).astype(bool)
    a = np.where(odd, o2, o0).astype(np.int64)
    b = np.where(odd, o3, o1).astype(np.int64)
    s = (a & 0xFFFF) + (a >> 16) + (b & 0xFFFF) + (b >> 16) - 2 * 65535
    return s.astype(np.int32)


def normal_f32(key, sub0, sub1, start, count, sigma) -> np.ndarray:
    s = irwin_hall_ints(key, sub0, sub1, start, count).astype(np.float32)  # exact
    return (s * sigma_const(sigma)).astype(np.float32)                     # one RNE multiply


def bf16_rne(v: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bits, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(v, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    return ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# --------------------------------------------------------------------------
# MXFP4 quantiser (input recipe; the oracle and the kernels only decode)
# --------------------------------------------------------------------------
def _floor_log2_f32(a: np.ndarray) -> np.ndarray:
    """Exact floor(log2(a)) for positive finite fp32 a (normal or subnormal)."""
    u = a.view(np.uint32)
    ef = ((u >> np.uint32(23)) & np.uint32(0xFF)).astype(np.int64)
    m = (u & np.uint32(0x7FFFFF)).astype(np.int64)
    # subnormal: value = m * 2^-149 -> floor(log2) = bit_length(m) - 150
    bl = np.zeros_like(m)
    mm = m.copy()
    for _ in range(23):
        nz = mm > 0
        bl += nz
        mm >>= 1
    return np.where(ef > 0, ef - 127, bl - 150)


def quantize_mxfp4(vals: np.ndarray):
    """Quantise fp32 rows [R][K] (K % 32 == 0) to (codes uint8 [R][K/2],
    scales uint8 [R][K/32]) as described in the module docstring."""
    vals = np.ascontiguousarray(vals, dtype=np.float32)
    R, K = vals.shape
    assert K % 32 == 0
    blk = vals.reshape(R, K // 32, 32)
    amax = np.abs(blk).max(axis=2)
    s = np.zeros(amax.shape, dtype=np.int64)
    pos = amax > 0
    s[pos] = _floor_log2_f32(amax[pos]) - 2 + 127
    s = np.clip(s, 0, 254)
    # 2^(127-s) as an exact fp32 (normal for s <= 253, subnormal 2^-127 at s = 254)
    ebits = (254 - s).astype(np.uint32)
    inv = np.where(ebits > 0, ebits << np.uint32(23), np.uint32(0x00400000)).astype(np.uint32).view(np.float32)
    a = (np.abs(blk) * inv[:, :, None]).astype(np.float32)
    mag = np.select(
        [a <= 0.25, a < 0.75, a <= 1.25, a < 1.75, a <= 2.5, a < 3.5, a <= 5.0],
        [0, 1, 2, 3, 4, 5, 6], default=7).astype(np.uint8)
    code = mag | np.where(np.signbit(blk), np.uint8(8), np.uint8(0)).astype(np.uint8)
    code = code.reshape(R, K)
    packed = (code[:, 0::2] | (code[:, 1::2] << np.uint8(4))).astype(np.uint8)
    return packed, s.astype(np.uint8)


# --------------------------------------------------------------------------
# Workloads
# --------------------------------------------------------------------------
@dataclass(frozen=True)
class MoEConfig:
    name: str
    hidden: int
    n_experts: int
    top_k: int
    inter: int
    shared_inter: int
    batch: int
    seed: int
    zipf_s: float = 0.0          # > 0: per-expert router bias -s*ln(rank)
    n_layers: int = 1
    n_steps: int = 1
    router_sigma: float = 0.05
    expert_sigma: float = 0.02
    shared_sigma: float = 0.02
    act_sigma: float = 1.0
    min_gap: float = 1e-3        # logit gap between the k-th and (k+1)-th expert
    scoring: str = "softmax"     # "sigmoid": the gap is taken on sigmoid(logit) + bias
    shared_format: str = "bf16"  # "mxfp4": the shared expert quantised like the routed ones
    verify_corr: float = 0.0     # > 0: a batch is `batch` positions of one sequence (see gen_tokens)

    def with_(self, **kw) -> "MoEConfig":
        return replace(self, **kw)

    # bytes the algorithm must move per layer-step (see the measurement notes)
    def expert_bytes(self) -> int:
        H, I = self.hidden, self.inter
        return 2 * I * (H // 2 + H // 32) + H * (I // 2 + I // 32)

    def counted_bytes(self, n_active: int) -> int:
        H = self.hidden
        shared = 3 * self.shared_inter * H * 2
        router = H * self.n_experts * 2
        acts = 3 * self.batch * H * 2
        return n_active * self.expert_bytes() + shared + router + acts


BASE_SEED = 20261202

CONFIGS = {
    0: MoEConfig("tiny_b1", 256, 32, 4, 128, 128, 1, BASE_SEED + 0),
    1: MoEConfig("full_b1", 7168, 896, 16, 2048, 2048, 1, BASE_SEED + 1),
    2: MoEConfig("full_b8", 7168, 896, 16, 2048, 2048, 8, BASE_SEED + 2),
    3: MoEConfig("full_b64_zipf", 7168, 896, 16, 2048, 2048, 64, BASE_SEED + 3, zipf_s=1.1),
    4: MoEConfig("full_stack4_b1", 7168, 896, 16, 2048, 2048, 1, BASE_SEED + 4,
                 n_layers=4, n_steps=64),
    # speculative-decoding verify step: 8 positions of one sequence (a token
    # and its drafts), whose activations share most of their direction
    5: MoEConfig("full_b8_verify", 7168, 896, 16, 2048, 2048, 8, BASE_SEED + 5, verify_corr=0.9),
}


# --------------------------------------------------------------------------
# Host generation
# --------------------------------------------------------------------------
def gen_bf16(cfg: MoEConfig, layer: int, tensor: int, shape, sigma, sub0=0, sub1=0):
    n = int(np.prod(shape))
    return bf16_rne(normal_f32(stream_key(cfg.seed, layer, tensor), sub0, sub1, 0, n, sigma)).reshape(shape)


def gen_router_w(cfg, layer=0):
    """bf16 [H][E] (element (h, e) is draw h*E + e)."""
    return gen_bf16(cfg, layer, T_ROUTER_W, (cfg.hidden, cfg.n_experts), cfg.router_sigma)


def gen_shared(cfg, layer=0):
    Is, H = cfg.shared_inter, cfg.hidden
    gu = gen_bf16(cfg, layer, T_SHARED_GU, (2 * Is, H), cfg.shared_sigma)
    d = gen_bf16(cfg, layer, T_SHARED_D, (H, Is), cfg.shared_sigma)
    return gu, d


def gen_expert(cfg, expert: int, layer=0):
    """MXFP4 tensors of one expert: gate/up codes [2I][H/2], scales [2I][H/32];
    down codes [H][I/2], scales [H][I/32].  Rows 0..I-1 of gate/up are gate."""
    H, I = cfg.hidden, cfg.inter
    gu = normal_f32(stream_key(cfg.seed, layer, T_EXPERT_GU), expert, 0, 0, 2 * I * H,
                    cfg.expert_sigma).reshape(2 * I, H)
    d = normal_f32(stream_key(cfg.seed, layer, T_EXPERT_D), expert, 0, 0, H * I,
                   cfg.expert_sigma).reshape(H, I)
    gc, gs = quantize_mxfp4(gu)
    dc, ds = quantize_mxfp4(d)
    return gc, gs, dc, ds


def gen_experts(cfg, experts, layer=0):
    """Stacked MXFP4 tensors for the listed experts (slot i = experts[i])."""
    parts = [gen_expert(cfg, int(e), layer) for e in experts]
    return tuple(np.stack([p[i] for p in parts]) for i in range(4))


def gen_router_bias(cfg, layer=0):
    """Zipf(s) log-prior per expert: bias_e = -s * ln(rank_e), rank a seeded
    permutation of 1..E (ranks ordered by Philox keys, ties by expert id).
    Returns None when the workload has no skew."""
    if cfg.zipf_s <= 0:
        return None
    E = cfg.n_experts
    o0, _, _, _ = philox4x32_10(np.arange(E, dtype=np.uint64), 0, 0, 0,
                                *stream_key(cfg.seed, layer, T_ZIPF_PERM))
    order = np.lexsort((np.arange(E), o0))           # experts by ascending key
    rank = np.empty(E, dtype=np.int64)
    rank[order] = np.arange(1, E + 1)
    return (-cfg.zipf_s * np.log(rank.astype(np.float64))).astype(np.float32)


def _logit_gap(x_bf16_row, wr_f64, bias, k, scoring="softmax"):
    lg = bf16_to_f32(x_bf16_row).astype(np.float64) @ wr_f64
    if scoring == "sigmoid":
        lg = 1.0 / (1.0 + np.exp(-lg))
    if bias is not None:
        lg = lg + bias.astype(np.float64)
    if k >= lg.shape[0]:
        return np.inf            # every expert is selected
    srt = np.sort(lg)[::-1]
    return srt[k - 1] - srt[k]


def gen_tokens(cfg, router_w_bf16, bias, token_ids, layer=0, max_attempts=64, tiny_every=0, tiny_exp=-30):
    """bf16 activations x [len(token_ids)][H].  Token t is drawn from
    substream (X, layer; sub0 = t, sub1 = attempt); a draw whose fp64 router
    logits (plus bias) put less than cfg.min_gap between the k-th and
    (k+1)-th largest is redrawn with the next attempt number, so that the
    selected expert set is decided with margin (input conditioning only;
    with cfg.scoring == "sigmoid" the margin is on sigmoid(logit) + bias).
    cfg.verify_corr = c > 0 makes a batch the positions of one sequence:
    x = sqrt(c) * (the sequence's draw) + sqrt(1 - c) * (the token's draw),
    in fp32, before the rounding (so the positions route to overlapping
    experts, as a speculative-decoding verify step does).
    tiny_every > 0 multiplies every tiny_every-th element of each draw by
    2^tiny_exp (exact in fp32) before the bf16 rounding, so that a row mixes
    elements some 2^30 apart in magnitude."""
    key = stream_key(cfg.seed, layer, T_X)
    wr = bf16_to_f32(router_w_bf16).astype(np.float64)
    out = np.empty((len(token_ids), cfg.hidden), dtype=np.uint16)
    attempts = np.zeros(len(token_ids), dtype=np.int32)
    c_base = np.float32(math.sqrt(cfg.verify_corr))
    c_own = np.float32(math.sqrt(1.0 - cfg.verify_corr))
    for i, t in enumerate(token_ids):
        base = None
        if cfg.verify_corr > 0:
            # positions of one sequence: token t is position t % batch of
            # sequence t // batch; all share that sequence's draw (sub1 = 2^20)
            base = normal_f32(key, int(t) // cfg.batch, 1 << 20, 0, cfg.hidden, cfg.act_sigma)
        for a in range(max_attempts):
            v = normal_f32(key, int(t), a, 0, cfg.hidden, cfg.act_sigma)
            if base is not None:
                v = (c_base * base + c_own * v).astype(np.float32)
            if tiny_every > 0:
                v[::tiny_every] *= np.float32(2.0 ** tiny_exp)
            row = bf16_rne(v)
            if _logit_gap(row, wr, bias, cfg.top_k, cfg.scoring) >= cfg.min_gap:
                break
        else:
            raise RuntimeError(f"no draw with logit gap >= {cfg.min_gap} for token {t}")
        out[i] = row
        attempts[i] = a
    return out, attempts


def gen_residual(cfg, token_ids, layer=0):
    key = stream_key(cfg.seed, layer, T_RESIDUAL)
    return np.stack([bf16_rne(normal_f32(key, int(t), 0, 0, cfg.hidden, cfg.act_sigma))
                     for t in token_ids])


def gen_tied_router(cfg, n_copies=4, with_bias=True, layer=0):
    """Router inputs whose logits tie exactly: bf16 Wr [H][E] with entries in
    {-1, 0, 1}, where the E columns come in groups of n_copies identical
    copies scattered over the expert ids (expert e belongs to group
    perm[e] mod E/n_copies, perm a seeded permutation), and an fp32 bias in
    {-2, ..., 2} per group, or None.  With integer activations every logit
    is an integer of magnitude <= H + 2, exact in fp32 and fp64 whatever
    the order of the sum.  Returns (router_w bits, bias, group)."""
    E, H = cfg.n_experts, cfg.hidden
    if E % n_copies:
        raise ValueError("n_experts must be a multiple of n_copies")
    G = E // n_copies
    key = stream_key(cfg.seed, layer, T_TIES)
    o0, o1, _, _ = philox4x32_10(np.arange(E, dtype=np.uint64), 0, 0, 0, *key)
    perm = np.lexsort((np.arange(E), o0))
    group = np.empty(E, dtype=np.int64)
    group[perm] = np.arange(E) % G
    c0, _, _, _ = philox4x32_10(np.arange(H * G, dtype=np.uint64), 1, 0, 0, *key)
    base = (c0.astype(np.int64) % 3 - 1).reshape(H, G).astype(np.float32)
    wr = bf16_rne(base[:, group])
    bias = None
    if with_bias:
        bg = (o1[:G].astype(np.int64) % 5 - 2).astype(np.float32)
        bias = bg[group]
    return wr, bias, group


def gen_tied_tokens(cfg, B, layer=0):
    """bf16 activations [B][H] with entries in {-1, 0, 1} (token 0 all zero,
    so its logits are the bias alone)."""
    H = cfg.hidden
    key = stream_key(cfg.seed, layer, T_TIES)
    c0, _, _, _ = philox4x32_10(np.arange(B * H, dtype=np.uint64), 2, 0, 0, *key)
    x = (c0.astype(np.int64) % 3 - 1).reshape(B, H).astype(np.float32)
    x[0] = 0.0
    return bf16_rne(x)


def gen_edge_mxfp4(cfg, n_experts, rows, K, tensor, s_lo, s_hi, zero_every=23, layer=0):
    """MXFP4 tensors that reach the format's corners: codes uint8
    [n_experts][rows][K/2] and scales uint8 [n_experts][rows][K/32].  Every
    32-element block holds each of the 16 E2M1 codes (negative zero, code 8,
    included) exactly twice, in a seeded order; scale bytes are drawn evenly
    from [s_lo, s_hi], and every zero_every-th block (counted over the whole
    tensor) gets s = 0, the smallest E8M0 value 2^-127.  Substream (EDGE,
    layer; sub0 = tensor)."""
    assert K % 32 == 0 and 0 <= s_lo <= s_hi <= 254
    key = stream_key(cfg.seed, layer, T_EDGE)
    nblk = n_experts * rows * (K // 32)
    n = nblk * 32
    o0, o1, _, _ = philox4x32_10(np.arange(n, dtype=np.uint64), int(tensor), 0, 0, *key)
    order = np.argsort(o0.reshape(nblk, 32), axis=1, kind="stable")
    codes = (order % 16).astype(np.uint8).reshape(n_experts, rows, K)
    packed = (codes[..., 0::2] | (codes[..., 1::2] << np.uint8(4))).astype(np.uint8)
    sb, _, _, _ = philox4x32_10(np.arange(nblk, dtype=np.uint64), int(tensor), 1, 0, *key)
    s = (s_lo + sb.astype(np.int64) % (s_hi - s_lo + 1)).astype(np.int64)
    if zero_every > 0:
        s[::zero_every] = 0
    return packed, s.astype(np.uint8).reshape(n_experts, rows, K // 32)


def gen_host_layer(cfg, layer=0, experts=None):
    """Everything for one layer on the host.  `experts` = list of expert ids
    to materialise (default: all, only sensible for small configs)."""
    if experts is None:
        experts = range(cfg.n_experts)
    experts = list(experts)
    wr = gen_router_w(cfg, layer)
    bias = gen_router_bias(cfg, layer)
    sgu, sd = gen_shared(cfg, layer)
    gc, gs, dc, ds = gen_experts(cfg, experts, layer)
    return dict(router_w=wr, router_bias=bias, shared_gu=sgu, shared_d=sd,
                gu_codes=gc, gu_scales=gs, d_codes=dc, d_scales=ds,
                experts=np.asarray(experts, dtype=np.int32))


# --------------------------------------------------------------------------
# Device generation (synth_gen.cu, same recipe, same bits)
# --------------------------------------------------------------------------
_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB = None


def lib_path() -> str:
    return os.path.join(_HERE, "libsynth.so")


def build(verbose=False) -> str:
    import subprocess
    src = os.path.join(_HERE, "synth_gen.cu")
    out = lib_path()
    cmd = ["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
           "-fmad=false", "-shared", "-Xcompiler", "-fPIC", "-o", out, src]
    if verbose:
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    return out


def _lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(lib_path()):
            raise RuntimeError("synth/libsynth.so is not built (run __graft_entry__.build())")
        L = ctypes.CDLL(lib_path())
        vp, u32, i64, f32 = ctypes.c_void_p, ctypes.c_uint32, ctypes.c_int64, ctypes.c_float
        L.synth_fill_bf16.argtypes = [vp, i64, u32, u32, u32, u32, f32, vp]
        L.synth_fill_mxfp4.argtypes = [vp, vp, i64, i64, i64, u32, u32, u32, f32, vp]
        L.synth_fill_bf16.restype = ctypes.c_int
        L.synth_fill_mxfp4.restype = ctypes.c_int
        _LIB = L
    return _LIB


def dev_fill_bf16(ptr: int, n: int, key, sub0: int, sub1: int, sigma: float, stream=0):
    rc = _lib().synth_fill_bf16(ptr, n, key[0], key[1], sub0, sub1, float(sigma_const(sigma)), stream)
    if rc != 0:
        raise RuntimeError(f"synth_fill_bf16 failed: {rc}")


def dev_fill_mxfp4(codes_ptr: int, scales_ptr: int, n_experts: int, rows: int, K: int,
                   key, expert0: int, sigma: float, stream=0):
    """Fill codes [n_experts][rows][K/2] and scales [n_experts][rows][K/32];
    slot i holds expert expert0 + i."""
    rc = _lib().synth_fill_mxfp4(codes_ptr, scales_ptr, n_experts, rows, K, key[0], key[1],
                                 expert0, float(sigma_const(sigma)), stream)
    if rc != 0:
        raise RuntimeError(f"synth_fill_mxfp4 failed: {rc}")
