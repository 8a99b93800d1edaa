"""ctypes binding of libcolimoe (include/coli_moe.h): argument marshalling only.

Every function here has the name of the C entry point it calls, takes torch
tensors that already live on the device (or None where the C call accepts
NULL), passes their data pointers and the current CUDA stream, and raises
``ColiError`` on a non-OK status.  No step of the layer runs in Python; if the
library is missing the import fails loudly.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libcolimoe.so")

# COLI_* constants of include/coli_moe.h
COLI_OK, COLI_ERR_INVALID_ARG, COLI_ERR_UNSUPPORTED, COLI_ERR_WORKSPACE = 0, 1, 2, 3
COLI_ERR_CUDA, COLI_ERR_NONFINITE, COLI_ERR_DEVICE = 4, 5, 6
COLI_FLAG_NONFINITE, COLI_FLAG_BAD_ID, COLI_FLAG_TIMEOUT, COLI_FLAG_RANGE = 0x1, 0x2, 0x4, 0x8
COLI_LAYER_PRENORM, COLI_PATH_DECODE, COLI_PATH_PREFILL = 0x1, 0x10, 0x20
COLI_LAYER_HOST_X, COLI_LAYER_HOST_OUT = 0x2, 0x4
COLI_FORM_DECODE_SPLITK, COLI_FORM_DECODE_TWOPHASE, COLI_FORM_PREFILL = 1, 2, 3

EXPORTS = ("coli_moe_route", "coli_moe_union", "coli_moe_expert_ffn", "coli_moe_layer",
           "coli_moe_workspace_bytes", "coli_moe_get_status", "coli_status_str", "coli_moe_version",
           "coli_moe_launch_count", "coli_moe_set_stage_events", "coli_moe_layer_noalloc", "coli_moe_ffn_form",
           "coli_moe_union_offsets", "coli_moe_test_wait_timeout", "coli_moe_layer_ep", "coli_moe_partial_to_bf16",
           "coli_moe_tier_state_bytes", "coli_moe_tier_reset", "coli_moe_layer_tiered", "coli_moe_tier_prefetch",
           "coli_moe_tier_lookahead")
COLI_NOALLOC_SCRATCH_BYTES = 32 << 20


class ColiError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_str(status)} (status {status})")
        self.status = status


class coli_moe_dims(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("inter", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("n_shared", ctypes.c_int32), ("group", ctypes.c_int32),
                ("code_bits", ctypes.c_int32)]


class coli_moe_weights(ctypes.Structure):
    _fields_ = [("gate_q", ctypes.c_void_p), ("up_q", ctypes.c_void_p), ("down_q", ctypes.c_void_p),
                ("gate_s", ctypes.c_void_p), ("up_s", ctypes.c_void_p), ("down_s", ctypes.c_void_p),
                ("router_w", ctypes.c_void_p), ("router_bias", ctypes.c_void_p)]


class coli_moe_tier(ctypes.Structure):
    _fields_ = [("gate_q", ctypes.c_void_p), ("up_q", ctypes.c_void_p), ("down_q", ctypes.c_void_p),
                ("gate_s", ctypes.c_void_p), ("up_s", ctypes.c_void_p), ("down_s", ctypes.c_void_p),
                ("n_slots", ctypes.c_int32), ("state", ctypes.c_void_p)]


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"{path} is not built; run `python -m int4_routed_expert_renorm_b200.build`")
    lib = ctypes.CDLL(path)
    P, I, Z, U32, U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_uint32, ctypes.c_uint64
    D, W = ctypes.POINTER(coli_moe_dims), ctypes.POINTER(coli_moe_weights)
    TR = ctypes.POINTER(coli_moe_tier)
    sig = {
        "coli_moe_route": (I, [P, P, I, I, I, P, P, P]),
        "coli_moe_union": (I, [P, I, I, I, P, P, P, P, P, P]),
        "coli_moe_expert_ffn": (I, [D, W, P, I, P, P, P, P, P, P, P, P, P, U32, P, Z, P]),
        "coli_moe_layer": (I, [D, W, P, I, P, P, U32, P, P, P, P, P, Z, P]),
        "coli_moe_workspace_bytes": (Z, [D, I]),
        "coli_moe_get_status": (I, [P, ctypes.POINTER(U32)]),
        "coli_status_str": (ctypes.c_char_p, [I]),
        "coli_moe_version": (I, []),
        "coli_moe_launch_count": (U64, [I]),
        "coli_moe_set_stage_events": (I, [ctypes.POINTER(ctypes.c_void_p), I]),
        "coli_moe_layer_noalloc": (I, [D, W, P, I, P, P, U32, P, P, P, P, P]),
        "coli_moe_ffn_form": (I, [D, I, U32, ctypes.POINTER(I)]),
        "coli_moe_union_offsets": (I, [D, I, ctypes.POINTER(Z)]),
        "coli_moe_test_wait_timeout": (I, [U64, P, P]),
        "coli_moe_layer_ep": (I, [D, W, I, I, I, P, I, P, P, U32, P, P, P, P, P, Z, P]),
        "coli_moe_partial_to_bf16": (I, [P, P, Z, P]),
        "coli_moe_tier_state_bytes": (Z, [D, I]),
        "coli_moe_tier_reset": (I, [D, TR, P]),
        "coli_moe_layer_tiered": (I, [D, W, TR, P, I, P, P, U32, P, P, P, P, P, Z, P]),
        "coli_moe_tier_prefetch": (I, [D, W, TR, P, I, P]),
        "coli_moe_tier_lookahead": (I, [D, W, TR, P, I, U32, P, Z, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype, f.argtypes = res, args
    return lib


_lib = load()


def status_str(s: int) -> str:
    return _lib.coli_status_str(s).decode()


def _ptr(t):
    """Device address of a tensor argument (None -> NULL).  The library reads and
    writes dense row-major device buffers, so only contiguous CUDA tensors pass:
    a strided view would be read as if it were dense, and a host pointer would
    reach a kernel."""
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensor arguments must be contiguous (dense, row-major)")
    if t.device.type != "cuda":
        raise ValueError(f"tensor arguments must be in device memory, got a tensor on {t.device}")
    return ctypes.c_void_p(t.data_ptr())


def _host_ptr(t, name: str):
    """Host address of a page-locked CPU tensor (COLI_LAYER_HOST_X / _OUT);
    the library maps it to its device address and refuses any other."""
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensor arguments must be contiguous (dense, row-major)")
    if t.device.type != "cpu" or not t.is_pinned():
        raise ValueError(f"{name}: the HOST flag needs a page-locked CPU tensor, got one on {t.device}")
    return ctypes.c_void_p(t.data_ptr())


def _need(t, n: int, esize: int, name: str, at_least: bool = False):
    """Refuse a tensor whose size does not match what the C call will read or
    write through its pointer (n elements of esize bytes; None passes)."""
    if t is None:
        return
    if t.element_size() != esize:
        raise ValueError(f"{name}: elements of {t.element_size()} bytes, the call needs {esize}")
    if (t.numel() < n) if at_least else (t.numel() != n):
        raise ValueError(f"{name}: {t.numel()} elements, the call needs {'at least ' if at_least else ''}{n}")


def _tokens(x, H: int) -> int:
    if x.dim() != 2 or x.shape[1] != H:
        raise ValueError(f"x: shape {tuple(x.shape)}, the call needs [T, {H}]")
    _need(x, x.shape[0] * H, 2, "x")
    return x.shape[0]


def _layer_sizes(dims, T: int, out, residual, logits_in, logits_out, topk_ids_out, topk_w_out):
    H, E, k = dims.hidden, dims.n_experts, dims.top_k
    _need(out, T * H, 2, "out")
    _need(residual, T * H, 2, "residual")
    _need(logits_in, T * E, 4, "logits_in")
    _need(logits_out, T * E, 4, "logits_out")
    _need(topk_ids_out, T * k, 4, "topk_ids_out")
    _need(topk_w_out, T * k, 4, "topk_w_out")


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(st: int, where: str):
    if st != COLI_OK:
        raise ColiError(st, where)


def coli_moe_version() -> int:
    return _lib.coli_moe_version()


def coli_moe_launch_count(reset: bool = False) -> int:
    return _lib.coli_moe_launch_count(1 if reset else 0)


def coli_moe_workspace_bytes(dims: coli_moe_dims, t_max: int) -> int:
    return _lib.coli_moe_workspace_bytes(ctypes.byref(dims), t_max)


def coli_moe_ffn_form(dims: coli_moe_dims, T: int, flags: int = 0) -> int:
    """The COLI_FORM_* value a layer call with these dims, T and flags takes
    (0 for T == 0); raises ColiError where the call would fail on them."""
    form = ctypes.c_int(0)
    _check(_lib.coli_moe_ffn_form(ctypes.byref(dims), T, flags, ctypes.byref(form)), "coli_moe_ffn_form")
    return form.value


def coli_moe_route(logits, bias, topk_ids, topk_w, stream=None):
    T, E = logits.shape
    k = topk_ids.shape[1]
    _need(logits, T * E, 4, "logits")
    _need(bias, E, 4, "bias")
    _need(topk_ids, T * k, 4, "topk_ids")
    _need(topk_w, T * k, 4, "topk_w")
    _check(_lib.coli_moe_route(_ptr(logits), _ptr(bias), T, E, k, _ptr(topk_ids), _ptr(topk_w), _stream(stream)),
           "coli_moe_route")


def coli_moe_union(topk_ids, n_experts, unique_ids, n_unique, seg_off, perm, pair_pos, stream=None):
    T, k = topk_ids.shape
    P = T * k
    _need(topk_ids, P, 4, "topk_ids")
    _need(unique_ids, min(n_experts, P), 4, "unique_ids", at_least=True)
    _need(n_unique, 1, 4, "n_unique", at_least=True)
    _need(seg_off, min(n_experts, P) + 1, 4, "seg_off", at_least=True)
    _need(perm, P, 4, "perm", at_least=True)
    _need(pair_pos, P, 4, "pair_pos", at_least=True)
    _check(_lib.coli_moe_union(_ptr(topk_ids), T, k, n_experts, _ptr(unique_ids), _ptr(n_unique), _ptr(seg_off),
                               _ptr(perm), _ptr(pair_pos), _stream(stream)), "coli_moe_union")


def coli_moe_expert_ffn(dims, weights, x, topk_ids, topk_w, unique_ids, n_unique, seg_off, perm, pair_pos,
                        residual, out, ws, flags=0, stream=None):
    T = _tokens(x, dims.hidden)
    P, E = T * dims.top_k, dims.n_experts
    _layer_sizes(dims, T, out, residual, None, None, topk_ids, topk_w)
    _need(unique_ids, min(E, P), 4, "unique_ids", at_least=True)
    _need(n_unique, 1, 4, "n_unique", at_least=True)
    _need(seg_off, min(E, P) + 1, 4, "seg_off", at_least=True)
    _need(perm, P, 4, "perm", at_least=True)
    _need(pair_pos, P, 4, "pair_pos", at_least=True)
    _check(_lib.coli_moe_expert_ffn(ctypes.byref(dims), ctypes.byref(weights), _ptr(x), T, _ptr(topk_ids),
                                    _ptr(topk_w), _ptr(unique_ids), _ptr(n_unique), _ptr(seg_off), _ptr(perm),
                                    _ptr(pair_pos), _ptr(residual), _ptr(out), flags, _ptr(ws),
                                    ws.numel() * ws.element_size(), _stream(stream)), "coli_moe_expert_ffn")


def _io_ptrs(flags, x, residual, out):
    """x, residual, out: device tensors, or page-locked CPU tensors under the
    COLI_LAYER_HOST_X (x, residual) and COLI_LAYER_HOST_OUT (out) flags."""
    hx, ho = flags & COLI_LAYER_HOST_X, flags & COLI_LAYER_HOST_OUT
    return ((_host_ptr(x, "x") if hx else _ptr(x)), (_host_ptr(residual, "residual") if hx else _ptr(residual)),
            (_host_ptr(out, "out") if ho else _ptr(out)))


def coli_moe_layer(dims, weights, x, out, ws, logits_in=None, residual=None, flags=0, logits_out=None,
                   topk_ids_out=None, topk_w_out=None, stream=None):
    T = _tokens(x, dims.hidden)
    _layer_sizes(dims, T, out, residual, logits_in, logits_out, topk_ids_out, topk_w_out)
    px, pr, po = _io_ptrs(flags, x, residual, out)
    _check(_lib.coli_moe_layer(ctypes.byref(dims), ctypes.byref(weights), px, T, _ptr(logits_in), pr, flags, po,
                               _ptr(logits_out), _ptr(topk_ids_out), _ptr(topk_w_out), _ptr(ws),
                               ws.numel() * ws.element_size(), _stream(stream)), "coli_moe_layer")


def coli_moe_layer_noalloc(dims, weights, x, out, logits_in=None, residual=None, flags=0, logits_out=None,
                           topk_ids_out=None, topk_w_out=None, stream=None):
    """coli_moe_layer with the library's own scratch instead of a workspace
    tensor, for callers that cannot allocate device memory (see the header)."""
    T = _tokens(x, dims.hidden)
    _layer_sizes(dims, T, out, residual, logits_in, logits_out, topk_ids_out, topk_w_out)
    px, pr, po = _io_ptrs(flags, x, residual, out)
    _check(_lib.coli_moe_layer_noalloc(ctypes.byref(dims), ctypes.byref(weights), px, T, _ptr(logits_in), pr, flags,
                                       po, _ptr(logits_out), _ptr(topk_ids_out), _ptr(topk_w_out),
                                       _stream(stream)), "coli_moe_layer_noalloc")


def coli_moe_layer_ep(dims, weights, expert_begin: int, expert_end: int, with_shared: bool, x, out_partial, ws,
                      logits_in=None, residual=None, flags=0, logits_out=None, topk_ids_out=None, topk_w_out=None,
                      stream=None):
    """One expert-parallel rank's fp32 partial output (see the header)."""
    T = _tokens(x, dims.hidden)
    _layer_sizes(dims, T, None, residual, logits_in, logits_out, topk_ids_out, topk_w_out)
    _need(out_partial, T * dims.hidden, 4, "out_partial")
    _check(_lib.coli_moe_layer_ep(ctypes.byref(dims), ctypes.byref(weights), expert_begin, expert_end,
                                  1 if with_shared else 0, _ptr(x), T, _ptr(logits_in), _ptr(residual), flags,
                                  _ptr(out_partial), _ptr(logits_out), _ptr(topk_ids_out), _ptr(topk_w_out), _ptr(ws),
                                  ws.numel() * ws.element_size(), _stream(stream)), "coli_moe_layer_ep")


def coli_moe_tier_state_bytes(dims, n_slots: int) -> int:
    return _lib.coli_moe_tier_state_bytes(ctypes.byref(dims), n_slots)


def coli_moe_tier_reset(dims, tier, stream=None):
    _check(_lib.coli_moe_tier_reset(ctypes.byref(dims), ctypes.byref(tier), _stream(stream)), "coli_moe_tier_reset")


def coli_moe_layer_tiered(dims, slots, tier, x, out, ws, logits_in=None, residual=None, flags=0, logits_out=None,
                          topk_ids_out=None, topk_w_out=None, stream=None):
    """coli_moe_layer through a host-RAM expert tier (see the header)."""
    T = _tokens(x, dims.hidden)
    _layer_sizes(dims, T, out, residual, logits_in, logits_out, topk_ids_out, topk_w_out)
    px, pr, po = _io_ptrs(flags, x, residual, out)
    _check(_lib.coli_moe_layer_tiered(ctypes.byref(dims), ctypes.byref(slots), ctypes.byref(tier), px, T,
                                      _ptr(logits_in), pr, flags, po, _ptr(logits_out), _ptr(topk_ids_out),
                                      _ptr(topk_w_out), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "coli_moe_layer_tiered")


def coli_moe_tier_prefetch(dims, slots, tier, ids, stream=None):
    """Places experts ids (device int32, at most n_slots of them) in the tier."""
    if ids.dtype.itemsize != 4:
        raise ValueError("ids: int32 expert ids")
    _check(_lib.coli_moe_tier_prefetch(ctypes.byref(dims), ctypes.byref(slots), ctypes.byref(tier), _ptr(ids),
                                       ids.numel(), _stream(stream)), "coli_moe_tier_prefetch")


def coli_moe_tier_lookahead(dims, next_slots, next_tier, x, ws, flags=0, stream=None):
    """Routes x with the next layer's router and places its experts in that
    layer's tier (see the header)."""
    T = _tokens(x, dims.hidden)
    _check(_lib.coli_moe_tier_lookahead(ctypes.byref(dims), ctypes.byref(next_slots), ctypes.byref(next_tier),
                                        _ptr(x), T, flags, _ptr(ws), ws.numel() * ws.element_size(),
                                        _stream(stream)), "coli_moe_tier_lookahead")


def coli_moe_partial_to_bf16(partial, out, stream=None):
    """out = bf16(partial), elementwise (out: bf16 bits, int16 tensor)."""
    n = partial.numel()
    _need(out, n, 2, "out")
    _check(_lib.coli_moe_partial_to_bf16(_ptr(partial), _ptr(out), n, _stream(stream)), "coli_moe_partial_to_bf16")


def coli_moe_union_offsets(dims, T: int) -> list[int]:
    """Byte offsets of unique_ids, n_unique, seg_off, perm and pair_pos inside
    the workspace of a coli_moe_layer call with these dims and T."""
    off = (ctypes.c_size_t * 5)()
    _check(_lib.coli_moe_union_offsets(ctypes.byref(dims), T, off), "coli_moe_union_offsets")
    return list(off)


def coli_moe_test_wait_timeout(limit_ns: int, elapsed=None, stream=None):
    """Test hook of the bounded device waits (see the header); elapsed: None or
    a device int64 tensor of 2 elements receiving each wait's duration in ns."""
    _need(elapsed, 2, 8, "elapsed")
    _check(_lib.coli_moe_test_wait_timeout(limit_ns, _ptr(elapsed), _stream(stream)), "coli_moe_test_wait_timeout")


def coli_moe_set_stage_events(events):
    """events: list of torch.cuda.Event (already recorded once, so they exist) or []."""
    n = len(events)
    arr = (ctypes.c_void_p * max(n, 1))(*[e.cuda_event for e in events])
    _check(_lib.coli_moe_set_stage_events(arr if n else None, n), "coli_moe_set_stage_events")


def coli_moe_get_status(stream=None):
    """Returns (status, flags); synchronises the stream and clears the device word."""
    f = ctypes.c_uint32(0)
    st = _lib.coli_moe_get_status(_stream(stream), ctypes.byref(f))
    return st, f.value
