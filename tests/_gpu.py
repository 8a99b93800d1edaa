"""Shared helpers of the GPU tests: device layers from the seeded generator and
the oracle's view of the same layer.  Nothing here computes the method."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import synth

needs_gpu = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")

# Tolerances derived from the arithmetic (kept next to the tests that use them):
#  * router weights: expf within 2 ulp per term, k terms summed in fp32 and one
#    division: |dw| <= (k + 4) * 2^-22 for weights in [0, 1];
#  * logits: fp32 dot product with at most ~40 rounding steps along any
#    summation path: |dl| <= 40 * 2^-24 * sum_h |x_h * w_h| (+ final rounding);
#  * layer output: max|gpu - ref| <= 1e-2 * max|ref| per output tensor (the
#    layer's stated bar), observed error reported alongside.
OUT_REL_TOL = 1e-2


def route_w_tol(k: int) -> float:
    return (k + 4) * 2.0 ** -22


def logits_tol(x_bits: np.ndarray, router_w: np.ndarray) -> np.ndarray:
    x = np.abs(synth.bf16_bits_to_f32(x_bits).astype(np.float64))
    return 40 * 2.0 ** -24 * (x @ np.abs(router_w.astype(np.float64)).T) + 1e-30


def device_layer(shape: synth.LayerShape, seed: int = 0, layer: int = 0):
    import synth.gpu as sg
    from int4_routed_expert_renorm_b200 import MoELayer, dims_for
    t = sg.expert_tensors(shape, seed, layer)
    li = synth.LayerInputs(shape, seed, layer)
    rw = torch.from_numpy(li.router_w()).cuda()
    b = li.bias()
    bias = None if b is None else torch.from_numpy(b).cuda()
    dims = dims_for(shape.hidden, shape.inter, shape.n_experts, shape.top_k, shape.n_shared, shape.group, shape.bits)
    return MoELayer(dims, t, rw, bias)


def oracle_weights(shape: synth.LayerShape, seed: int = 0, layer: int = 0, cache: int = 0):
    import oracle
    return oracle.ExpertWeights.from_synth(synth.LayerInputs(shape, seed, layer), cache=cache)


def bits(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint16)


def to_dev_bits(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def ambiguous_tokens(l32_ref: np.ndarray, tol: np.ndarray, bias, k: int) -> np.ndarray:
    """Tokens whose k-th / (k+1)-th logit gap is within twice the logit
    tolerance: their selection depends on rounding, so either choice is valid."""
    lb = l32_ref.astype(np.float64) + (0 if bias is None else bias.astype(np.float64)[None, :])
    s = -np.sort(-lb, axis=1)
    if lb.shape[1] <= k:
        return np.zeros(lb.shape[0], bool)
    gap = s[:, k - 1] - s[:, k]
    return gap <= 2 * tol.max(axis=1)
