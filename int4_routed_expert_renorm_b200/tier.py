"""Host-RAM expert tier for one layer: every routed expert in page-locked host
memory, `n_slots` of them on the device at a time (Place, Overlap, Learn; see
``coli_moe_tier`` in the header).  This module holds the tensors and
marshals arguments; placement, copies and the layer are the library's.
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from ._lib import (COLI_ERR_INVALID_ARG, ColiError, coli_moe_dims, coli_moe_layer_tiered, coli_moe_tier,
                   coli_moe_tier_lookahead, coli_moe_tier_prefetch, coli_moe_tier_reset, coli_moe_tier_state_bytes,
                   coli_moe_weights, coli_moe_workspace_bytes)

_NAMES = ("gate_q", "up_q", "down_q", "gate_s", "up_s", "down_s")


class TieredLayer:
    """One layer whose routed experts live in host memory.

    tensors: the whole layer's expert tensors (leading dimension E + S: the
    routed experts, then the shared ones), on the host or the device; the
    routed part is copied into page-locked host memory, the shared experts
    into the device slot arrays after the `n_slots` routed slots.
    """

    def __init__(self, dims: coli_moe_dims, tensors: dict, n_slots: int, router_w: torch.Tensor | None = None,
                 bias: torch.Tensor | None = None, device="cuda"):
        E, S = dims.n_experts, dims.n_shared
        if not 1 <= n_slots <= E:
            raise ValueError(f"n_slots {n_slots} outside [1, {E}]")
        self.dims, self.n_slots = dims, n_slots
        self.host, self.slots = {}, {}
        for name in _NAMES:
            t = tensors[name]
            if t.shape[0] != E + S or not t.is_contiguous():
                raise ValueError(f"{name}: {tuple(t.shape)}, needs a dense [E + S, ...] tensor")
            self.host[name] = t[:E].to("cpu").pin_memory()
            slot = torch.zeros((n_slots + S,) + tuple(t.shape[1:]), dtype=t.dtype, device=device)
            if S:
                slot[n_slots:].copy_(t[E:])
            self.slots[name] = slot
        self.router_w, self.bias = router_w, bias
        p = lambda x: None if x is None else ctypes.c_void_p(x.data_ptr())  # noqa: E731
        self.weights = coli_moe_weights(*(p(self.slots[n]) for n in _NAMES), p(router_w), p(bias))
        nbytes = coli_moe_tier_state_bytes(dims, n_slots)
        if nbytes == 0:
            raise ColiError(COLI_ERR_INVALID_ARG, "coli_moe_tier_state_bytes")
        self.state = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.tier = coli_moe_tier(*(p(self.host[n]) for n in _NAMES), n_slots, p(self.state))
        self.reset()

    def reset(self, stream=None):
        """Empty every slot; clear the usage counts and the counters."""
        coli_moe_tier_reset(self.dims, self.tier, stream)

    def workspace(self, t_max: int, device="cuda") -> torch.Tensor:
        return torch.empty(coli_moe_workspace_bytes(self.dims, t_max), dtype=torch.uint8, device=device)

    def forward(self, x, out, ws, **kw):
        coli_moe_layer_tiered(self.dims, self.weights, self.tier, x, out, ws, **kw)
        return out

    def prefetch(self, ids: torch.Tensor, stream=None):
        """Place experts `ids` (device int32, at most n_slots) ahead of use."""
        coli_moe_tier_prefetch(self.dims, self.weights, self.tier, ids.contiguous(), stream)

    def lookahead(self, x: torch.Tensor, ws: torch.Tensor, flags: int = 0, stream=None):
        """Route x (the previous layer's input, on the device) with this
        layer's router and place the experts it selects: run it on another
        stream while the previous layer computes.  `ws` is a workspace of its
        own (``workspace(T)``)."""
        coli_moe_tier_lookahead(self.dims, self.weights, self.tier, x, ws, flags, stream)

    # ---- Learn: the usage counts, kept across runs ----------------------------
    def usage(self) -> np.ndarray:
        """Routed pairs per expert over every call since the last reset."""
        return self.state_arrays()["usage"]

    def warm_from_usage(self, usage, stream=None):
        """Start from a saved usage profile (for example a previous run's
        ``usage()``): the counts are written into the tier's state and its
        ``n_slots`` most used experts (ties to the lower index) are placed, so
        that the hottest experts are resident before the first call."""
        E = self.dims.n_experts
        u = np.asarray(usage, dtype=np.int64).reshape(-1)
        if u.size != E or (u < 0).any():
            raise ValueError(f"usage: {u.size} non-negative counts needed, one per expert ({E})")
        u = np.minimum(u, 0xFFFFFFFF).astype(np.uint32)
        words = torch.from_numpy(u.view(np.int32).copy()).to(self.state.device)
        C = self.n_slots
        off = 4 * (E + C)                                   # usage[E] follows slot_of[E] and owner[C]
        torch.cuda.synchronize()
        self.state[off:off + 4 * E].copy_(words.view(torch.uint8))
        hot = np.lexsort((np.arange(E), -u.astype(np.int64)))[:C].astype(np.int32)
        self.prefetch(torch.from_numpy(hot).to(self.state.device), stream)

    # ---- the state, read back (synchronises) ------------------------------
    def _words(self) -> np.ndarray:
        torch.cuda.synchronize()
        return self.state.cpu().numpy().view(np.int32)

    def state_arrays(self) -> dict:
        """slot_of[E], owner[C], usage[E], last[C] and the counters."""
        E, C = self.dims.n_experts, self.n_slots
        w = self._words()
        return {"slot_of": w[:E].copy(), "owner": w[E:E + C].copy(),
                "usage": w[E + C:2 * E + C].view(np.uint32).copy(),
                "last": w[2 * E + C:2 * E + 2 * C].view(np.uint32).copy(),
                "calls": int(w[2 * E + 2 * C]), "hits": int(w[2 * E + 2 * C + 1]),
                "misses": int(w[2 * E + 2 * C + 2]), "fills": int(w[2 * E + 2 * C + 3])}
