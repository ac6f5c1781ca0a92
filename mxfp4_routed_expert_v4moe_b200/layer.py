"""MoELayer: holds device weights and buffers and calls the three C-ABI steps.

Allocation (weights, workspace, outputs) goes through torch; the computation
is entirely libv4moe's. Buffers are cached per token count so repeated calls
allocate nothing.
"""
from __future__ import annotations

import torch

from . import (check, make_config, make_weights, v4moe_forward, v4moe_layer, v4moe_permute,
               v4moe_route, v4moe_workspace_bytes)


class MoELayer:
    def __init__(self, *, H, I, E, k, Is, gate, w13_codes, w13_scales, w2_codes, w2_scales,
                 sh_w13=None, sh_w13_scale=None, sh_w2=None, sh_w2_scale=None, vocab=129280,
                 routed_scale=1.5, swiglu_limit=10.0):
        self.H, self.I, self.E, self.k, self.Is = H, I, E, k, Is
        self.cfg = make_config(H, I, E, k, Is, vocab, routed_scale, swiglu_limit)
        self.gate = gate
        self.tensors = dict(w13_codes=w13_codes, w13_scales=w13_scales, w2_codes=w2_codes,
                            w2_scales=w2_scales, sh_w13=sh_w13, sh_w13_scale=sh_w13_scale,
                            sh_w2=sh_w2, sh_w2_scale=sh_w2_scale)
        self.weights = make_weights(**self.tensors)
        self.device = gate.device
        self._bufs = {}
        self._ws = None

    @classmethod
    def from_host(cls, li, device="cuda"):
        """Upload a host description (numpy arrays with the generator's field names)."""
        wl = li.wl

        def up(a, dtype=None):
            if a is None:
                return None
            t = torch.from_numpy(a)
            if dtype is not None:
                t = t.view(dtype)
            return t.to(device).contiguous()

        return cls(H=wl.H, I=wl.I, E=wl.E, k=wl.k, Is=wl.Is, gate=up(li.gate, torch.bfloat16),
                   w13_codes=up(li.w13_codes), w13_scales=up(li.w13_scales),
                   w2_codes=up(li.w2_codes), w2_scales=up(li.w2_scales), sh_w13=up(li.sh13),
                   sh_w13_scale=up(li.sh13_scale), sh_w2=up(li.sh2), sh_w2_scale=up(li.sh2_scale),
                   vocab=wl.vocab if li.tid2eid is None else li.tid2eid.shape[0],
                   routed_scale=wl.routed_scale, swiglu_limit=wl.swiglu_limit)

    # -- buffers ---------------------------------------------------------------
    def workspace(self, T):
        need = v4moe_workspace_bytes(self.cfg, T)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.zeros(max(need, 256), dtype=torch.uint8, device=self.device)
        return self._ws

    def buffers(self, T):
        b = self._bufs.get(T)
        if b is None:
            d = self.device
            S = T * self.k
            b = dict(topk_ids=torch.empty((T, self.k), dtype=torch.int32, device=d),
                     topk_w=torch.empty((T, self.k), dtype=torch.float32, device=d),
                     counts=torch.empty(self.E, dtype=torch.int32, device=d),
                     offsets=torch.empty(self.E + 1, dtype=torch.int32, device=d),
                     sorted_slot=torch.empty(max(S, 1), dtype=torch.int32, device=d),
                     slot_pos=torch.empty(max(S, 1), dtype=torch.int32, device=d),
                     out=torch.empty((T, self.H), dtype=torch.bfloat16, device=d))
            self._bufs[T] = b
        return b

    # -- the three steps -------------------------------------------------------
    def route(self, x, bias=None, token_ids=None, tid2eid=None, stream=None):
        T = x.shape[0]
        b = self.buffers(T)
        ws = self.workspace(T)
        check(v4moe_route(self.cfg, T, x, self.gate, bias, token_ids, tid2eid, b["topk_ids"],
                          b["topk_w"], ws, ws.numel(), stream), "v4moe_route")
        return b["topk_ids"], b["topk_w"]

    def permute(self, topk_ids, stream=None):
        T = topk_ids.shape[0]
        b = self.buffers(T)
        ws = self.workspace(T)
        check(v4moe_permute(self.cfg, T, topk_ids, b["counts"], b["offsets"], b["sorted_slot"],
                            b["slot_pos"], ws, ws.numel(), stream), "v4moe_permute")
        return b["counts"], b["offsets"], b["sorted_slot"], b["slot_pos"]

    def forward(self, x, topk_ids, topk_w, offsets, sorted_slot, slot_pos, out=None, stream=None):
        T = x.shape[0]
        b = self.buffers(T)
        ws = self.workspace(T)
        out = b["out"] if out is None else out
        check(v4moe_forward(self.cfg, T, x, topk_ids, topk_w, offsets, sorted_slot, slot_pos,
                            self.weights, out, ws, ws.numel(), stream), "v4moe_forward")
        return out

    def __call__(self, x, bias=None, token_ids=None, tid2eid=None, out=None, stream=None):
        """The whole layer through v4moe_layer (routing outputs kept in buffers(T))."""
        T = x.shape[0]
        b = self.buffers(T)
        ws = self.workspace(T)
        out = b["out"] if out is None else out
        check(v4moe_layer(self.cfg, T, x, self.gate, bias, token_ids, tid2eid, self.weights,
                          b["topk_ids"], b["topk_w"], b["counts"], b["offsets"], b["sorted_slot"],
                          b["slot_pos"], out, ws, ws.numel(), stream), "v4moe_layer")
        return out
