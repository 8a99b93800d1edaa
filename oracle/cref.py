"""The plain-C oracle (``oracle/c/moe_ref.c``) through ctypes -- TEST INFRASTRUCTURE.

Only ``tests/`` import this module (and ``__graft_entry__.build()`` compiles the
library).  The C oracle is a second, independent statement of the layer that
``oracle/moe.py`` states: the same readings of the pages, written from the
definitions in plain C with double arithmetic.  The two are checked against
each other and against the same pins in ``tests/test_oracle_c.py``.

    python -m oracle.cref          # compile oracle/libcolimoeref.so with gcc
"""
from __future__ import annotations

import contextlib
import ctypes as C
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "c", "moe_ref.c")
LIB = os.path.join(HERE, "libcolimoeref.so")
CC = os.environ.get("CC", "gcc")
CFLAGS = ["-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math", "-Wall", "-Wextra", "-shared", "-fPIC"]

_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle if its library is missing or older than the source."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = f"{LIB}.{os.getpid()}.tmp"       # concurrent test processes each build their own, then rename
        r = subprocess.run([CC, *CFLAGS, SRC, "-o", tmp, "-lm"], capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"{CC} failed for the C oracle:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, LIB)
    return LIB


def _load():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
    return _lib


@contextlib.contextmanager
def using(path: str):
    """Route every call to the library at ``path`` (a build of a modified copy
    of the source, for the mutation tests) while the block runs."""
    global _lib
    saved, _lib = _load(), C.CDLL(path)
    try:
        yield
    finally:
        _lib = saved


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _call(name, *args):
    rc = getattr(_load(), name)(*args)
    if rc != 0:
        raise ValueError(f"{name}: status {rc}")


def _arr(a, dt):
    return np.ascontiguousarray(np.asarray(a, dtype=dt))


def decode_fp16(bits) -> np.ndarray:
    b = _arr(bits, np.uint16)
    out = np.empty(b.shape, np.float64)
    _call("coli_ref_decode", C.c_long(b.size), _p(b), 0, _p(out))
    return out


def decode_bf16(bits) -> np.ndarray:
    b = _arr(bits, np.uint16)
    out = np.empty(b.shape, np.float64)
    _call("coli_ref_decode", C.c_long(b.size), _p(b), 1, _p(out))
    return out


def round_bf16(v) -> np.ndarray:
    a = _arr(v, np.float64)
    out = np.empty(a.shape, np.float64)
    _call("coli_ref_round_bf16", C.c_long(a.size), _p(a), _p(out), None)
    return out


def f64_to_bf16_bits(v) -> np.ndarray:
    a = _arr(v, np.float64)
    out = np.empty(a.shape, np.uint16)
    _call("coli_ref_round_bf16", C.c_long(a.size), _p(a), None, _p(out))
    return out


def dequant(q, s, group: int = 32, bits: int = 4) -> np.ndarray:
    q, s = _arr(q, np.uint8), _arr(s, np.uint16)
    rows, K = q.shape[0], q.shape[1] * 8 // bits
    if s.shape != (rows, K // group):
        raise ValueError("scale shape")
    out = np.empty((rows, K), np.float64)
    _call("coli_ref_dequant", rows, K, group, bits, _p(q), _p(s), _p(out))
    return out


def router_logits(x_bits, router_w):
    x, wr = _arr(x_bits, np.uint16), _arr(router_w, np.float32)
    T, H = x.shape
    E = wr.shape[0]
    l64, l32 = np.empty((T, E), np.float64), np.empty((T, E), np.float32)
    _call("coli_ref_router_logits", T, E, H, _p(x), _p(wr), _p(l64), _p(l32))
    return l64, l32


def route(l32, k: int, bias=None):
    l = _arr(l32, np.float32)
    T, E = l.shape
    b = None if bias is None else _arr(bias, np.float32)
    ids, w, flags = np.empty((T, k), np.int32), np.empty((T, k), np.float64), np.empty(T, np.int32)
    _call("coli_ref_route", T, E, k, _p(l), _p(b), _p(ids), _p(w), _p(flags))
    return ids, w, flags


def batch_union(ids, n_experts: int):
    flat = _arr(ids, np.int32).reshape(-1)
    P = flat.size
    unique, seg = np.empty(n_experts, np.int32), np.empty(n_experts + 1, np.int32)
    perm, pos, nu = np.empty(max(P, 1), np.int32), np.empty(max(P, 1), np.int32), np.zeros(1, np.int32)
    _call("coli_ref_union", P, n_experts, _p(flat), _p(unique), _p(nu), _p(seg), _p(perm), _p(pos))
    U = int(nu[0])
    return unique[:U].copy(), seg[:U + 1].copy(), perm[:P].copy(), pos[:P].copy()


def rms_norm(h_bits) -> np.ndarray:
    h = _arr(h_bits, np.uint16)
    out = np.empty_like(h)
    _call("coli_ref_rms_norm", h.shape[0], h.shape[1], _p(h), _p(out))
    return out


def moe_layer(arrays: dict, x_bits, n_experts: int, top_k: int, n_shared: int, group: int = 32, bits: int = 4,
              router_w=None, bias=None, logits_in=None, residual_bits=None) -> dict:
    """One layer with every expert resident.  ``arrays`` = {'gate': (codes,
    scales), 'up': ..., 'down': ...}, each with a leading axis of
    n_experts + n_shared.  Returns dict(logits64, logits32, ids, w, flags, acc, out)."""
    x = _arr(x_bits, np.uint16)
    T, H = x.shape
    gq, gs = (_arr(a, t) for a, t in zip(arrays["gate"], (np.uint8, np.uint16)))
    uq, us = (_arr(a, t) for a, t in zip(arrays["up"], (np.uint8, np.uint16)))
    dq, ds = (_arr(a, t) for a, t in zip(arrays["down"], (np.uint8, np.uint16)))
    n, I = gq.shape[0], gq.shape[1]
    if n != n_experts + n_shared or dq.shape[:2] != (n, H) or gq.shape[2] * 8 // bits != H:
        raise ValueError("expert array shapes")
    E, k = n_experts, top_k
    rw = None if router_w is None else _arr(router_w, np.float32)
    li = None if logits_in is None else _arr(logits_in, np.float32)
    b = None if bias is None else _arr(bias, np.float32)
    res = None if residual_bits is None else _arr(residual_bits, np.uint16)
    r = dict(logits64=np.empty((T, E)), logits32=np.empty((T, E), np.float32), ids=np.empty((T, k), np.int32),
             w=np.empty((T, k)), flags=np.empty(T, np.int32), acc=np.empty((T, H)), out=np.empty((T, H), np.uint16))
    _call("coli_ref_moe_layer", T, H, I, E, k, n_shared, group, bits, _p(gq), _p(gs), _p(uq), _p(us), _p(dq),
          _p(ds), _p(x), _p(rw), _p(li), _p(b), _p(res), _p(r["logits64"]), _p(r["logits32"]), _p(r["ids"]),
          _p(r["w"]), _p(r["flags"]), _p(r["acc"]), _p(r["out"]))
    return r


def moe_layer_experts(fetch, hidden: int, inter: int, x_bits, n_experts: int, top_k: int, n_shared: int,
                      group: int = 32, bits: int = 4, router_w=None, bias=None, logits_in=None,
                      residual_bits=None, experts=None) -> dict:
    """The layer with experts fetched on demand: ``fetch(kind, e)`` returns
    (codes, scales) of expert e for kind 'gate', 'up' or 'down'.  The batch is
    routed first (the C oracle's logits and Route) to learn which routed
    experts it selects; only those and the shared experts are fetched, or the
    ids in ``experts`` when given (the call fails if one it needs is missing).
    Returns what ``moe_layer`` returns."""
    x = _arr(x_bits, np.uint16)
    T = x.shape[0]
    E, k, n = n_experts, top_k, n_experts + n_shared
    li = None if logits_in is None else _arr(logits_in, np.float32)
    l32 = li if li is not None else router_logits(x, router_w)[1]
    ids = route(l32, k, bias)[0]
    need = sorted(set(ids.ravel().tolist()) | set(range(E, n))) if experts is None else sorted(experts)
    held = {(kind, e): tuple(_arr(a, t) for a, t in zip(fetch(kind, e), (np.uint8, np.uint16)))
            for kind in ("gate", "up", "down") for e in need}
    ptrs = {}
    for kind in ("gate", "up", "down"):
        q, sc = (C.c_void_p * n)(), (C.c_void_p * n)()
        for e in need:
            q[e], sc[e] = held[(kind, e)][0].ctypes.data, held[(kind, e)][1].ctypes.data
        ptrs[kind] = (q, sc)
    rw = None if router_w is None else _arr(router_w, np.float32)
    b = None if bias is None else _arr(bias, np.float32)
    res = None if residual_bits is None else _arr(residual_bits, np.uint16)
    r = dict(logits64=np.empty((T, E)), logits32=np.empty((T, E), np.float32), ids=np.empty((T, k), np.int32),
             w=np.empty((T, k)), flags=np.empty(T, np.int32), acc=np.empty((T, hidden)),
             out=np.empty((T, hidden), np.uint16))
    _call("coli_ref_moe_layer_experts", T, hidden, inter, E, k, n_shared, group, bits, *ptrs["gate"], *ptrs["up"],
          *ptrs["down"], _p(x), _p(rw), _p(li), _p(b), _p(res), _p(r["logits64"]), _p(r["logits32"]),
          _p(r["ids"]), _p(r["w"]), _p(r["flags"]), _p(r["acc"]), _p(r["out"]))
    return r


if __name__ == "__main__":
    print("built", build(force=True))
