"""Device side of the seeded input generator: fills expert weight tensors in
device memory with the same SplitMix64 streams as ``synth`` (numpy).

Input generation only.  Uses ``synth/libcolisynth.so`` (built by
``python -m int4_routed_expert_renorm_b200.build``).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

from . import (DOWN_Q, DOWN_S, GATE_Q, GATE_S, UP_Q, UP_S, LayerInputs, LayerShape, activations,
               stream_key)

_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libcolisynth.so")
        if not os.path.exists(path):
            raise ImportError(f"{path} is not built")
        lib = ctypes.CDLL(path)
        for n in ("coli_synth_fill_codes", "coli_synth_fill_scales"):
            f = getattr(lib, n)
            f.restype = ctypes.c_int
            f.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_void_p, ctypes.c_void_p]
        _LIB = lib
    return _LIB


def fill_codes(t: torch.Tensor, key: int, start: int = 0):
    st = torch.cuda.current_stream().cuda_stream
    r = _lib().coli_synth_fill_codes(key, start, t.numel(), ctypes.c_void_p(t.data_ptr()), ctypes.c_void_p(st))
    if r != 0:
        raise RuntimeError(f"coli_synth_fill_codes failed ({r})")


def fill_scales(t: torch.Tensor, key: int, start: int = 0):
    st = torch.cuda.current_stream().cuda_stream
    r = _lib().coli_synth_fill_scales(key, start, t.numel(), ctypes.c_void_p(t.data_ptr()), ctypes.c_void_p(st))
    if r != 0:
        raise RuntimeError(f"coli_synth_fill_scales failed ({r})")


def expert_tensors(shape: LayerShape, seed: int = 0, layer: int = 0, device="cuda") -> dict:
    """All E+S experts' codes and scales of one layer, on the device.

    Returns {'gate_q','up_q','down_q': uint8, 'gate_s','up_s','down_s': int16 (fp16 bits)}."""
    H, I, n = shape.hidden, shape.inter, shape.n_total
    out = {}
    for name, kind, (r, K) in (("gate", GATE_Q, (I, H)), ("up", UP_Q, (I, H)), ("down", DOWN_Q, (H, I))):
        q = torch.empty((n, r, K * shape.bits // 8), dtype=torch.uint8, device=device)
        fill_codes(q, stream_key(seed, layer, kind))
        out[name + "_q"] = q
    for name, kind, (r, K) in (("gate", GATE_S, (I, H)), ("up", UP_S, (I, H)), ("down", DOWN_S, (H, I))):
        s = torch.empty((n, r, K // shape.group), dtype=torch.int16, device=device)
        fill_scales(s, stream_key(seed, layer, kind))
        out[name + "_s"] = s
    return out


def dense_inputs(shape: LayerShape, seed: int = 0, layer: int = 0, batch: int = 0, device="cuda") -> dict:
    """Router weight / bias / logits and the bf16 activations of one layer, on the device."""
    li = LayerInputs(shape, seed, layer)
    d = {"x": torch.from_numpy(activations(shape, seed, batch).view(np.int16)).to(device)}
    if shape.logits_in:
        d["logits"] = torch.from_numpy(li.logits()).to(device)
    else:
        d["router_w"] = torch.from_numpy(li.router_w()).to(device)
    b = li.bias()
    d["bias"] = None if b is None else torch.from_numpy(b).to(device)
    return d
