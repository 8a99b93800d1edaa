"""Holder for one MoE layer's device tensors and the C structs that describe them.

Argument marshalling only: ``MoELayer.forward`` is one ``coli_moe_layer`` call.
"""
from __future__ import annotations

import ctypes

import torch

from ._lib import (COLI_ERR_INVALID_ARG, COLI_ERR_UNSUPPORTED, ColiError, coli_moe_dims, coli_moe_layer,
                   coli_moe_weights, coli_moe_workspace_bytes)


def dims_for(hidden: int, inter: int, n_experts: int, top_k: int, n_shared: int, group: int = 32,
             code_bits: int = 4) -> coli_moe_dims:
    return coli_moe_dims(hidden, inter, n_experts, top_k, n_shared, group, code_bits)


class MoELayer:
    """Device tensors of one layer: gate/up/down codes (uint8) and fp16 scale
    bits (int16 tensors), router weight fp32 [E, H] (optional) and bias fp32 [E]
    (optional), in the container layout of ``include/coli_moe.h``."""

    def __init__(self, dims: coli_moe_dims, tensors: dict, router_w: torch.Tensor | None = None,
                 bias: torch.Tensor | None = None):
        self.dims = dims
        self.t = dict(tensors)
        H, I, G = dims.hidden, dims.inter, dims.group
        n = dims.n_experts + dims.n_shared
        cb = 8 if dims.code_bits == 8 else 4
        want = {"gate_q": (n, I, H * cb // 8), "up_q": (n, I, H * cb // 8), "down_q": (n, H, I * cb // 8),
                "gate_s": (n, I, H // G), "up_s": (n, I, H // G), "down_s": (n, H, I // G)}
        for name, shp in want.items():
            if self.t[name].numel() != shp[0] * shp[1] * shp[2]:
                raise ValueError(f"{name}: {self.t[name].numel()} elements, the dims need {shp}")
        self.router_w = router_w
        self.bias = bias
        held = [self.t[name] for name in want] + [v for v in (router_w, bias) if v is not None]
        if not all(v.is_contiguous() for v in held):
            raise ValueError("weight tensors must be contiguous (dense, row-major)")
        self._on_device = all(v.device.type == "cuda" for v in held)
        p = lambda x: None if x is None else ctypes.c_void_p(x.data_ptr())  # noqa: E731
        self.weights = coli_moe_weights(p(self.t["gate_q"]), p(self.t["up_q"]), p(self.t["down_q"]),
                                        p(self.t["gate_s"]), p(self.t["up_s"]), p(self.t["down_s"]),
                                        p(router_w), p(bias))

    def workspace(self, t_max: int, device="cuda") -> torch.Tensor:
        """Scratch for any call of up to ``t_max`` tokens; raises ColiError for
        dims the library does not support or a negative ``t_max``."""
        n = coli_moe_workspace_bytes(self.dims, t_max)
        if n == 0:
            raise ColiError(COLI_ERR_INVALID_ARG if t_max < 0 else COLI_ERR_UNSUPPORTED, "coli_moe_workspace_bytes")
        return torch.empty(n, dtype=torch.uint8, device=device)

    def forward(self, x: torch.Tensor, out: torch.Tensor, ws: torch.Tensor, logits_in=None, residual=None,
                flags: int = 0, logits_out=None, topk_ids_out=None, topk_w_out=None, stream=None):
        if not self._on_device:
            raise ValueError("the layer's weight tensors must be in device memory")
        coli_moe_layer(self.dims, self.weights, x, out, ws, logits_in=logits_in, residual=residual, flags=flags,
                       logits_out=logits_out, topk_ids_out=topk_ids_out, topk_w_out=topk_w_out, stream=stream)
        return out
