"""Expert parallelism: one layer's experts spread over several GPUs.

Each rank holds a contiguous range of the routed experts (the rank that holds
the shared experts also adds the residual).  Every rank routes the whole batch
over all experts (the router is replicated) and computes its experts' share of
the output with ``coli_moe_layer_ep``; an all-reduce over the ranks sums the
fp32 shares, and ``coli_moe_partial_to_bf16`` rounds the sum once.  This
module marshals arguments and issues the collective; the computation is the
library's.
"""
from __future__ import annotations

import ctypes

import torch

from ._lib import (COLI_ERR_INVALID_ARG, COLI_ERR_UNSUPPORTED, ColiError, coli_moe_dims, coli_moe_layer_ep,
                   coli_moe_partial_to_bf16, coli_moe_weights, coli_moe_workspace_bytes)

_NAMES = ("gate_q", "up_q", "down_q", "gate_s", "up_s", "down_s")


def expert_range(n_experts: int, rank: int, world: int) -> tuple[int, int]:
    """Rank `rank` of `world`'s contiguous share [begin, end) of the routed
    experts: sizes differ by at most one, every expert belongs to one rank."""
    if world < 1 or not 0 <= rank < world or n_experts < world:
        raise ValueError(f"cannot split {n_experts} experts over rank {rank} of {world}")
    return rank * n_experts // world, (rank + 1) * n_experts // world


def local_tensors(tensors: dict, dims: coli_moe_dims, begin: int, end: int, with_shared: bool) -> dict:
    """A rank's expert tensors cut from the whole layer's (leading dimension =
    expert): routed experts [begin, end), then the shared ones if it holds them."""
    E, S = dims.n_experts, dims.n_shared
    out = {}
    for name in _NAMES:
        t = tensors[name]
        parts = [t[begin:end]] + ([t[E:E + S]] if with_shared and S else [])
        out[name] = torch.cat(parts).contiguous()
    return out


def allreduce_partial(partial: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the ranks' fp32 partial outputs in place (no-op without a process
    group of more than one rank)."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(partial, op=dist.ReduceOp.SUM, group=group)
    return partial


class ExpertParallelLayer:
    """One rank's share of a layer: its experts' device tensors (as cut by
    ``local_tensors``), the full router weight fp32 [E, H] and bias fp32 [E]."""

    def __init__(self, dims: coli_moe_dims, tensors: dict, begin: int, end: int, with_shared: bool,
                 router_w: torch.Tensor | None = None, bias: torch.Tensor | None = None):
        if not 0 <= begin < end <= dims.n_experts:
            raise ValueError(f"expert range [{begin}, {end}) outside [0, {dims.n_experts})")
        self.dims, self.begin, self.end, self.with_shared = dims, begin, end, with_shared
        self.t = dict(tensors)
        H, I, G = dims.hidden, dims.inter, dims.group
        n = (end - begin) + (dims.n_shared if with_shared else 0)
        cb = 8 if dims.code_bits == 8 else 4
        want = {"gate_q": (n, I, H * cb // 8), "up_q": (n, I, H * cb // 8), "down_q": (n, H, I * cb // 8),
                "gate_s": (n, I, H // G), "up_s": (n, I, H // G), "down_s": (n, H, I // G)}
        for name, shp in want.items():
            if self.t[name].numel() != shp[0] * shp[1] * shp[2]:
                raise ValueError(f"{name}: {self.t[name].numel()} elements, this rank's experts need {shp}")
        held = [self.t[name] for name in want] + [v for v in (router_w, bias) if v is not None]
        if not all(v.is_contiguous() for v in held):
            raise ValueError("weight tensors must be contiguous (dense, row-major)")
        self.router_w, self.bias = router_w, bias
        p = lambda x: None if x is None else ctypes.c_void_p(x.data_ptr())  # noqa: E731
        self.weights = coli_moe_weights(p(self.t["gate_q"]), p(self.t["up_q"]), p(self.t["down_q"]),
                                        p(self.t["gate_s"]), p(self.t["up_s"]), p(self.t["down_s"]),
                                        p(router_w), p(bias))

    def workspace(self, t_max: int, device="cuda") -> torch.Tensor:
        n = coli_moe_workspace_bytes(self.dims, t_max)
        if n == 0:
            raise ColiError(COLI_ERR_INVALID_ARG if t_max < 0 else COLI_ERR_UNSUPPORTED, "coli_moe_workspace_bytes")
        return torch.empty(n, dtype=torch.uint8, device=device)

    def partial(self, x: torch.Tensor, partial: torch.Tensor, ws: torch.Tensor, logits_in=None, residual=None,
                flags: int = 0, logits_out=None, topk_ids_out=None, topk_w_out=None, stream=None) -> torch.Tensor:
        """This rank's fp32 share of the output; the residual is added on the
        rank that holds the shared experts only."""
        coli_moe_layer_ep(self.dims, self.weights, self.begin, self.end, self.with_shared, x, partial, ws,
                          logits_in=logits_in, residual=residual if self.with_shared else None, flags=flags,
                          logits_out=logits_out, topk_ids_out=topk_ids_out, topk_w_out=topk_w_out, stream=stream)
        return partial

    def forward(self, x: torch.Tensor, out: torch.Tensor, ws: torch.Tensor, partial: torch.Tensor, group=None,
                **kw) -> torch.Tensor:
        """The layer's output (bf16 bits in `out`) on every rank: this rank's
        share, the all-reduce of the shares over `group`, one rounding."""
        self.partial(x, partial, ws, **kw)
        allreduce_partial(partial, group)
        coli_moe_partial_to_bf16(partial, out)
        return out
