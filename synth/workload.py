"""Device-resident synthetic workloads (torch tensors on the GPU) built with
the seeded generator, plus host copies of the parts the oracle needs.
Inputs only: nothing here computes any step of the MoE layer."""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from . import (T_EXPERT_D, T_EXPERT_GU, T_ROUTER_W, T_SHARED_D, T_SHARED_GU, T_SHARED_MX_D, T_SHARED_MX_GU,
               MoEConfig,
               dev_fill_bf16, dev_fill_mxfp4, gen_edge_mxfp4, gen_residual, gen_router_bias, gen_tokens,
               stream_key)


def _t():
    import torch
    return torch


def to_host_u16(t) -> np.ndarray:
    torch = _t()
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def u16_to_device(a: np.ndarray, device="cuda"):
    torch = _t()
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).to(device).view(torch.bfloat16)


@dataclass
class DeviceLayer:
    cfg: MoEConfig
    layer: int
    router_w: object      # bf16 [H][E]
    router_bias: object   # fp32 [E] or None
    gu_codes: object      # u8 [E][2I][H/2]
    gu_scales: object     # u8 [E][2I][H/32]
    d_codes: object       # u8 [E][H][I/2]
    d_scales: object      # u8 [E][H][I/32]
    shared_gu: object     # bf16 [2Is][H]
    shared_d: object      # bf16 [H][Is]
    router_w_host: np.ndarray
    bias_host: np.ndarray | None
    shared_mx: tuple | None = None   # MXFP4 shared expert: (gu codes, gu scales, d codes, d scales)

    def host_experts(self, experts):
        """Host copies of the listed experts' packed tensors (slot order)."""
        torch = _t()
        idx = torch.as_tensor(np.asarray(experts, dtype=np.int64), device=self.gu_codes.device)
        return tuple(t.index_select(0, idx).cpu().numpy() for t in
                     (self.gu_codes, self.gu_scales, self.d_codes, self.d_scales))

    def host_shared(self):
        if self.shared_gu is None:
            return None, None
        return to_host_u16(self.shared_gu), to_host_u16(self.shared_d)

    def host_shared_mx(self):
        return None if self.shared_mx is None else tuple(t.cpu().numpy() for t in self.shared_mx)

    def weights_struct(self):
        from sparse_moe_decode_router_b200.api import moe_layer_weights
        p = lambda t: None if t is None else t.data_ptr()
        mx = self.shared_mx if self.shared_mx is not None else (None,) * 4
        return moe_layer_weights(p(self.router_w), p(self.router_bias), p(self.gu_codes), p(self.gu_scales),
                                 p(self.d_codes), p(self.d_scales), p(self.shared_gu), p(self.shared_d),
                                 *(p(t) for t in mx))

    def tokens(self, token_ids, tiny_every=0):
        """bf16 x for the given token ids (gap-conditioned), host and device;
        tiny_every > 0: every tiny_every-th element scaled by 2^-30."""
        x, _ = gen_tokens(self.cfg, self.router_w_host, self.bias_host, list(token_ids), layer=self.layer,
                          tiny_every=tiny_every)
        return x, u16_to_device(x, self.gu_codes.device)


def make_device_layer(cfg: MoEConfig, layer: int = 0, device="cuda") -> DeviceLayer:
    torch = _t()
    H, E, I, Is = cfg.hidden, cfg.n_experts, cfg.inter, cfg.shared_inter
    dev = torch.device(device)
    gu_c = torch.empty((E, 2 * I, H // 2), dtype=torch.uint8, device=dev)
    gu_s = torch.empty((E, 2 * I, H // 32), dtype=torch.uint8, device=dev)
    d_c = torch.empty((E, H, I // 2), dtype=torch.uint8, device=dev)
    d_s = torch.empty((E, H, I // 32), dtype=torch.uint8, device=dev)
    dev_fill_mxfp4(gu_c.data_ptr(), gu_s.data_ptr(), E, 2 * I, H, stream_key(cfg.seed, layer, T_EXPERT_GU), 0,
                   cfg.expert_sigma)
    dev_fill_mxfp4(d_c.data_ptr(), d_s.data_ptr(), E, H, I, stream_key(cfg.seed, layer, T_EXPERT_D), 0,
                   cfg.expert_sigma)
    wr = torch.empty((H, E), dtype=torch.bfloat16, device=dev)
    dev_fill_bf16(wr.data_ptr(), H * E, stream_key(cfg.seed, layer, T_ROUTER_W), 0, 0, cfg.router_sigma)
    sgu = sd = smx = None
    if Is > 0 and cfg.shared_format == "mxfp4":
        smx = (torch.empty((1, 2 * Is, H // 2), dtype=torch.uint8, device=dev),
               torch.empty((1, 2 * Is, H // 32), dtype=torch.uint8, device=dev),
               torch.empty((1, H, Is // 2), dtype=torch.uint8, device=dev),
               torch.empty((1, H, Is // 32), dtype=torch.uint8, device=dev))
        dev_fill_mxfp4(smx[0].data_ptr(), smx[1].data_ptr(), 1, 2 * Is, H, stream_key(cfg.seed, layer, T_SHARED_MX_GU),
                       0, cfg.shared_sigma)
        dev_fill_mxfp4(smx[2].data_ptr(), smx[3].data_ptr(), 1, H, Is, stream_key(cfg.seed, layer, T_SHARED_MX_D),
                       0, cfg.shared_sigma)
        smx = tuple(t[0] for t in smx)
    elif Is > 0:
        sgu = torch.empty((2 * Is, H), dtype=torch.bfloat16, device=dev)
        sd = torch.empty((H, Is), dtype=torch.bfloat16, device=dev)
        dev_fill_bf16(sgu.data_ptr(), 2 * Is * H, stream_key(cfg.seed, layer, T_SHARED_GU), 0, 0, cfg.shared_sigma)
        dev_fill_bf16(sd.data_ptr(), H * Is, stream_key(cfg.seed, layer, T_SHARED_D), 0, 0, cfg.shared_sigma)
    bias_host = gen_router_bias(cfg, layer)
    bias = None if bias_host is None else torch.from_numpy(bias_host).to(dev)
    torch.cuda.synchronize(dev)
    return DeviceLayer(cfg, layer, wr, bias, gu_c, gu_s, d_c, d_s, sgu, sd, to_host_u16(wr), bias_host, smx)


def residual_tokens(cfg: MoEConfig, token_ids, layer: int = 0, device="cuda"):
    r = gen_residual(cfg, list(token_ids), layer)
    return r, u16_to_device(r, device)


def with_edge_experts(dl: DeviceLayer, gu_scales=(87, 139), d_scales=(115, 167)) -> DeviceLayer:
    """The same layer with every routed expert replaced by corner-case MXFP4
    tensors (synth.gen_edge_mxfp4): all 16 E2M1 codes in every block, scale
    bytes spread over the given ranges (defaults: gate/up 2^-40 .. 2^12, down
    2^-12 .. 2^40, chosen so that the layer's outputs stay inside fp32) and a
    share of s = 0 blocks.  Router, shared expert and seeds are unchanged."""
    import dataclasses
    torch = _t()
    c = dl.cfg
    H, E, I = c.hidden, c.n_experts, c.inter
    gc, gs = gen_edge_mxfp4(c, E, 2 * I, H, T_EXPERT_GU, *gu_scales, layer=dl.layer)
    dc, ds = gen_edge_mxfp4(c, E, H, I, T_EXPERT_D, *d_scales, layer=dl.layer)
    dev = dl.gu_codes.device
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    return dataclasses.replace(dl, gu_codes=to(gc), gu_scales=to(gs), d_codes=to(dc), d_scales=to(ds))
