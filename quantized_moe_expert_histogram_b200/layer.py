"""One quantised MoE layer driven through the C ABI.

``QuantMoELayer`` owns device buffers (plumbing: torch allocates them) and
runs the path call by call: moe_route_permute (router, optional bit gate,
permutation) -> moe_grouped_ffn_combine (grouped FFN and weighted
combine).  No arithmetic happens here.
"""
from __future__ import annotations

import torch

from . import moeq


class QuantMoELayer:
    def __init__(self, d, E, k, F, group, layout, w_router, bias, blobs, max_tokens, device="cuda",
                 w_bit=None, bias_bit=None):
        self.d, self.E, self.k, self.F, self.group = d, E, k, F, group
        self.layout = layout
        self.w_router = w_router
        self.bias = bias
        # optional bit-width gate (nested-plane layout): widths chosen per
        # (token, selected expert) on the device by moe_bit_gate
        self.w_bit, self.bias_bit = w_bit, bias_bit
        self.blobs = blobs
        self.device = torch.device(device)
        self.max_tokens = max_tokens
        self._alloc(max_tokens)

    @classmethod
    def from_weights(cls, shape, w_router, bias, w_gate, w_up, w_down, max_tokens, device="cuda"):
        layout = moeq.LAYOUT_PLANES if shape.layout == "planes" else moeq.LAYOUT_INT4
        blobs = moeq.moe_quant_pack(w_gate, w_up, w_down, shape.group, layout)
        return cls(shape.d, shape.E, shape.k, shape.F, shape.group, layout, w_router, bias, blobs,
                   max_tokens, device)

    def _alloc(self, T):
        dev, k, d = self.device, self.k, self.d
        nb = self.E * (3 if self.layout == moeq.LAYOUT_PLANES else 1)
        rows = T * k
        self.buf = dict(
            topk_idx=torch.empty(T, k, dtype=torch.int32, device=dev),
            topk_w=torch.empty(T, k, dtype=torch.float32, device=dev),
            counts=torch.empty(nb, dtype=torch.int32, device=dev),
            offsets=torch.empty(nb + 1, dtype=torch.int32, device=dev),
            perm=torch.empty(rows, dtype=torch.int32, device=dev),
            inv_perm=torch.empty(rows, dtype=torch.int32, device=dev),
            x_perm=torch.empty(rows, d, dtype=torch.float16, device=dev),
            y_perm=torch.empty(rows, d, dtype=torch.float16, device=dev),
            workspace=torch.empty(max(16, moeq.moe_ffn_workspace_bytes(rows, self.E, d, self.F, self.layout),
                                      moeq.moe_ffn_combine_workspace_bytes(T, k, self.E, d, self.F, self.layout)),
                                  dtype=torch.uint8, device=dev),
            y=torch.empty(T, d, dtype=torch.bfloat16, device=dev),
            bits=torch.empty(T, k, dtype=torch.uint8, device=dev),
            status=torch.zeros(1, dtype=torch.int32, device=dev),
            route_ws=torch.empty(max(256, moeq.moe_route_workspace_bytes(T, d, self.E)), dtype=torch.uint8,
                                 device=dev),
            perm_ws=torch.empty(moeq.moe_permute_workspace_bytes(T, self.E, k, self.layout == moeq.LAYOUT_PLANES),
                                dtype=torch.uint8, device=dev),
            rp_ws=torch.empty(moeq.moe_route_permute_workspace_bytes(T, d, self.E, k,
                                                                     self.layout == moeq.LAYOUT_PLANES),
                              dtype=torch.uint8, device=dev),
        )

    def views(self, T):
        b, k = self.buf, self.k
        rows = T * k
        return dict(topk_idx=b["topk_idx"][:T], topk_w=b["topk_w"][:T], counts=b["counts"],
                    offsets=b["offsets"], perm=b["perm"][:rows], inv_perm=b["inv_perm"][:rows],
                    x_perm=b["x_perm"][:rows], y_perm=b["y_perm"][:rows], workspace=b["workspace"],
                    y=b["y"][:T], status=b["status"], route_ws=b["route_ws"], perm_ws=b["perm_ws"],
                    rp_ws=b["rp_ws"], bits=b["bits"][:T])

    def forward(self, x, bits=None, forced_idx=None, residual=None, stream=None):
        """One layer pass.  ``bits`` (uint8 [T,k], nested layout) fixes the
        widths; when it is None and the layer has a bit gate, the widths come
        from moe_bit_gate on the device."""
        T = x.shape[0]
        if T > self.max_tokens:
            raise ValueError(f"T={T} exceeds max_tokens={self.max_tokens}")
        v = self.views(T)
        gate = bits is None and self.w_bit is not None
        moeq.moe_route_permute(x, self.w_router, self.bias, self.k, forced_idx=forced_idx, bits=bits,
                               w_bit=self.w_bit if gate else None, bias_bit=self.bias_bit if gate else None,
                               out=v, status=v["status"], workspace=v["rp_ws"], stream=stream)
        moeq.moe_grouped_ffn_combine(v["x_perm"], v["offsets"], self.blobs, T, self.k, self.E, self.d, self.F,
                                     self.group, self.layout, v["perm"], v["inv_perm"], v["topk_w"],
                                     residual=residual, y=v["y"], y_perm=v["y_perm"], workspace=v["workspace"],
                                     status=v["status"], stream=stream)
        return v["y"]
