"""Decode through an expert bank larger than the GPU's budget (caller-side loop).

Expert paging keeps a stable logical expert index while the weights move
between a pinned host bank and HBM slots ("Running MoE LLMs on a single GPU:
what expert offloading actually costs", section "Inside expert paging"); the
experts the next layer's router would pick for the current hidden state are
prefetched while the current layer computes (FloE verdict page, JSON field
referee_report.summary, point iii).  This module only sequences calls into the
C library: routing, permutation, the grouped FFN and the combine run in its
kernels, the replacement policy and copies in its expert cache.  The host
reads each layer's expert indices to form the need set (one device-to-host
copy per layer).

Per layer l of one decode step:
  1. route x_l with layer l's router (moe_route_topk) and permute;
  2. optionally (`prefetch_top`), predict layer l+1's experts from x_l with
     layer l+1's router and issue the prefetch of each token's most likely
     ones (copies overlap this layer's FFN on the cache's stream);
  3. read the need set; in waves of at most slots_per_layer experts:
     moe_cache_lookup -> moe_grouped_ffn through the slot map -> release;
  4. combine; x_{l+1} = x_l + out_l (residual).
Each layer's input is the hidden state scaled to unit RMS per token (a
pre-norm without learned weights): without it the stack's residual stream,
fed through 48 random SwiGLU layers, grows until it overflows.
"""
from __future__ import annotations

import ctypes
from typing import Dict, List, Optional

import numpy as np
import torch

from . import _native as N

_ALIGN = 256


def _al(n: int) -> int:
    return (n + _ALIGN - 1) // _ALIGN * _ALIGN


class ExpertBlob:
    """Byte layout of one expert in the bank and in an HBM slot."""

    def __init__(self, experts: Dict[str, torch.Tensor]):
        self.parts = [k for k in ("w13", "s13", "w2", "s2") if k in experts]
        self.nbytes = {k: experts[k][0].numel() * experts[k].element_size() for k in self.parts}
        self.offset = {}
        o = 0
        for k in self.parts:
            self.offset[k] = o
            o = _al(o + self.nbytes[k])
        self.size = o


class OffloadedBank:
    """n_layers MoE layers whose routed experts live in the cache's pinned host bank."""

    def __init__(self, shape, n_layers: int, slots_per_layer: int, T: int, device=0):
        self.shape, self.L, self.C, self.T = shape, n_layers, slots_per_layer, T
        self.dev = torch.device("cuda", device)
        self.blob: Optional[ExpertBlob] = None
        self.cache: Optional[N.ExpertCache] = None
        self.routers: List[torch.Tensor] = [None] * n_layers
        self.biases: List[Optional[torch.Tensor]] = [None] * n_layers
        self.gscales: List[Dict[str, torch.Tensor]] = [{} for _ in range(n_layers)]
        self.desc = N.make_desc(shape, T)
        ws_bytes = N.moe_workspace_size(self.desc)
        E, k, d = shape.n_experts, shape.top_k, shape.d_model
        self.ws = torch.empty(ws_bytes, dtype=torch.uint8, device=self.dev)
        self.ws_pred = torch.empty(ws_bytes, dtype=torch.uint8, device=self.dev)
        self.idx = torch.empty(T, k, dtype=torch.int32, device=self.dev)
        self.gw = torch.empty(T, k, dtype=torch.float32, device=self.dev)
        self.idx_pred = torch.empty(T, k, dtype=torch.int32, device=self.dev)
        self.gw_pred = torch.empty(T, k, dtype=torch.float32, device=self.dev)
        self.offs = torch.empty(E + 1, dtype=torch.int32, device=self.dev)
        self.rtok = torch.empty(T * k, dtype=torch.int32, device=self.dev)
        self.inv = torch.empty(T * k, dtype=torch.int32, device=self.dev)
        self.y = torch.empty(T * k, d, dtype=torch.bfloat16, device=self.dev)
        self.slot_map = torch.full((E,), -1, dtype=torch.int32, device=self.dev)
        self.trace: List[tuple] = []
        # experts prefetched per token: its prefetch_top highest-scoring
        # predictions for the next layer (0: no prefetch, the default; None:
        # every prediction when the predicted set fits in a quarter of the
        # layer's slots, else each token's most likely one).  Measured on the
        # 48-layer NVFP4 bank with 25% of the experts resident, in steady
        # state, the stack is bound by the host-to-device copies at 1, 4 and
        # 16 tokens per step, and a prefetch hides no copy time: it only adds
        # the bytes of predictions that go unused (about 17% of them) and
        # evicts experts the layer was about to use, so no prefetch was faster
        # at every batch size.  With faster copies or more slots than the need
        # set the overlap would pay, hence the option.
        self.prefetch_top = 0

    # -------------------------------------------------------------- filling
    def fill_layer(self, l: int, layer: Dict[str, object]):
        """Copy layer l's router, offsets and experts (a moe_inputs layer draw) into the bank."""
        ex = layer["experts"]
        if self.blob is None:
            self.blob = ExpertBlob(ex)
            self.cache = N.ExpertCache(self.L, self.shape.n_experts, self.C, self.blob.size, self.dev.index)
        self.routers[l] = layer["router"].to(self.dev)
        self.biases[l] = layer["bias"].to(self.dev) if layer.get("bias") is not None else None
        for key in ("g13", "g2"):
            if key in ex:
                self.gscales[l][key] = ex[key].to(self.dev).contiguous()
        E = self.shape.n_experts
        for e in range(E):
            base = self.cache.host_expert(l, e)
            for key in self.blob.parts:
                src = ex[key][e].contiguous()
                nb = self.blob.nbytes[key]
                buf = (ctypes.c_uint8 * nb).from_address(base + self.blob.offset[key])
                dst = torch.frombuffer(buf, dtype=torch.uint8)
                dst.copy_(src.reshape(-1).view(torch.uint8).cpu() if src.device.type != "cpu"
                          else src.reshape(-1).view(torch.uint8))

    def slot_weights(self, l: int) -> N.Weights:
        base = self.cache.slot_base(l)
        w = N.Weights()
        for key in self.blob.parts:
            setattr(w, key, base + self.blob.offset[key])
        w.g13 = N._ptr(self.gscales[l].get("g13"))
        w.g2 = N._ptr(self.gscales[l].get("g2"))
        w.stride_w13 = w.stride_s13 = w.stride_w2 = w.stride_s2 = self.blob.size
        w.slot_map = self.slot_map.data_ptr()
        w.n_physical = self.C
        return w

    # -------------------------------------------------------------- running
    def forward_layer(self, l: int, x: torch.Tensor, out: torch.Tensor, prefetch: bool = True, stream=None):
        st = stream or torch.cuda.current_stream(self.dev)
        d = self.desc
        N.moe_route_topk(d, x, self.routers[l], self.biases[l], self.idx, self.gw, self.ws, st)
        N.moe_permute(d, self.idx, self.offs, self.rtok, self.inv, st)
        if prefetch and self.prefetch_top != 0 and l + 1 < self.L:
            N.moe_route_topk(d, x, self.routers[l + 1], self.biases[l + 1], self.idx_pred, self.gw_pred,
                             self.ws_pred, st)
            # each token's selection is in descending logit order
            sel = self.idx_pred.cpu().numpy()
            depth = self.prefetch_top
            if depth is None:
                depth = sel.shape[1] if np.unique(sel).size <= self.C // 4 else 1
            pred = np.unique(sel[:, :depth])
            self.trace.append(("prefetch", l + 1, pred.tolist()))
            self.cache.prefetch(l + 1, pred)
        need = np.unique(self.idx.cpu().numpy()).tolist()
        w = self.slot_weights(l)
        for w0 in range(0, len(need), self.C):
            wave = need[w0: w0 + self.C]
            self.trace.append(("lookup", l, wave))
            self.cache.lookup(l, wave, self.slot_map, st)
            N.moe_grouped_ffn(d, w, None, self.offs, self.rtok, x, self.y, None, self.ws, st)
            self.cache.release(l, st)
        N.moe_combine(d, self.y, self.inv, self.gw, None, out, st)

    def decode_step(self, x0: torch.Tensor, prefetch: bool = True, keep: bool = False):
        """All layers on one batch: x_{l+1} = x_l + out_l, layer l applied to x_l
        scaled to unit RMS per token.  Returns the last hidden state (and every
        layer's input and output when keep=True)."""
        x = x0
        ins, outs = [], []
        for l in range(self.L):
            xf = x.float()
            xin = (xf * torch.rsqrt(xf.pow(2).mean(dim=1, keepdim=True) + 1e-6)).to(torch.bfloat16)
            out = torch.empty_like(x)
            self.forward_layer(l, xin, out, prefetch=prefetch)
            if keep:
                ins.append(xin)
                outs.append(out)
            x = (xf + out.float()).to(torch.bfloat16)
        return (x, ins, outs) if keep else x

    def stats(self) -> dict:
        return self.cache.stats()

    def close(self):
        if self.cache is not None:
            self.cache.close()
            self.cache = None
