"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in the oracle (on the CPU, by monkeypatching a
copy of one function) and checks that at least one pin of
``test_oracle_pins.py`` fails.  Nothing here touches a GPU.
"""
import numpy as np
import pytest

import oracle
import oracle.moe as M
import tests.test_oracle_pins as P

PINS = [getattr(P, n) for n in dir(P) if n.startswith("test_") and n not in (
    "test_batch_union_brute_force_and_invariants",)]


def _union_pin():
    for T, E, k in [(4, 16, 2), (33, 40, 3), (64, 256, 8)]:
        P.test_batch_union_brute_force_and_invariants(T, E, k)


def _some_pin_fails():
    for f in PINS + [_union_pin]:
        try:
            f()
        except Exception:  # noqa: BLE001 - any failure counts as caught
            return True
    return False


def _swap_nibbles(q):
    b = np.asarray(q, dtype=np.uint8)
    nib = np.empty(b.shape[:-1] + (b.shape[-1] * 2,), dtype=np.int16)
    nib[..., 0::2] = b >> 4
    nib[..., 1::2] = b & 0x0F
    return (nib - 16 * (nib >= 8)).astype(np.int8)


def _offset_codes(q):
    b = np.asarray(q, dtype=np.uint8)
    nib = np.empty(b.shape[:-1] + (b.shape[-1] * 2,), dtype=np.int16)
    nib[..., 0::2] = b & 0x0F
    nib[..., 1::2] = b >> 4
    return (nib - 8).astype(np.int8)


def _interleaved_scales(q_bytes, s_bits, group=32):
    q = M.unpack_int4(q_bytes).astype(np.float64)
    s = M.fp16_bits_to_f64(s_bits)
    rows, k = q.shape
    return (q.reshape(rows, group, k // group) * s[:, None, :]).reshape(rows, k)


def _scale_per_32_codes(q_bytes, s_bits, group=32):
    """Every scale applied to 32 codes whatever the group, the row's tail
    keeping the last scale."""
    q = M.unpack_int4(q_bytes).astype(np.float64)
    s = M.fp16_bits_to_f64(s_bits)
    idx = np.minimum(np.arange(q.shape[1]) // 32, s.shape[1] - 1)
    return q * s[:, idx]


def _int8_unsigned(q_bytes):
    return np.asarray(q_bytes, dtype=np.uint8).astype(np.int16)


def _route_high_index_ties(l32, k):
    l = np.asarray(l32, dtype=np.float32).astype(np.float64)
    T, E = l.shape
    key = np.where(np.isnan(l), -np.inf, l)
    idx = np.broadcast_to(np.arange(E), (T, E))
    order = np.lexsort((-idx, -key), axis=1)
    ids = order[:, :k].astype(np.int32)
    sel = np.take_along_axis(key, order[:, :k], axis=1)
    e = np.exp(sel - sel[:, :1])
    return ids, e / e.sum(1, keepdims=True), np.zeros(T, np.int64)


def _route_not_renormalised(l32, k):
    ids, w, f = ORIG["route"](l32, k)
    l = np.asarray(l32, np.float64)
    p = np.exp(l - l.max(1, keepdims=True))
    p = p / p.sum(1, keepdims=True)
    return ids, np.take_along_axis(p, ids.astype(np.int64), 1), f


def _union_unstable(ids, n_experts):
    u, s, perm, pp = ORIG["batch_union"](ids, n_experts)
    for a, b in zip(s[:-1], s[1:]):
        perm[a:b] = perm[a:b][::-1]
    pp = np.empty_like(perm)
    pp[perm] = np.arange(perm.size, dtype=np.int32)
    return u, s, perm, pp


def _ffn_no_h_round(W, e, x64):
    g = x64 @ W.matrix("gate", e).T
    u = x64 @ W.matrix("up", e).T
    return (M.silu(g) * u) @ W.matrix("down", e).T


def _ffn_gate_up_swapped(W, e, x64):
    g = x64 @ W.matrix("up", e).T
    u = x64 @ W.matrix("gate", e).T
    return M.round_bf16(M.silu(g) * u) @ W.matrix("down", e).T


def _combine_drop(what):
    def f(W, x_bits, ids, w, n_experts, n_shared, residual_bits=None, return_f64=False):
        if what == "shared":
            n_shared = 0
        if what == "residual":
            residual_bits = None
        if what == "weights":
            w = np.ones_like(np.asarray(w, dtype=np.float64))
        return ORIG["moe_ffn_combine"](W, x_bits, ids, w, n_experts, n_shared, residual_bits, return_f64)
    return f


def _rms_no_sqrt(h_bits):
    h = M.bf16_bits_to_f64(h_bits)
    return M.f64_to_bf16_bits(h / (np.mean(h * h, axis=1, keepdims=True) + M.RMS_EPS))


def _silu_as_sigmoid(g):
    return 1.0 / (1.0 + np.exp(-g))


def _round_via_fp32(v):
    return np.asarray(v, np.float64).astype(np.float32).astype(np.float64).round(6)


def _round_ties_away(v):
    v = np.asarray(v, np.float64)
    out = v.copy()
    fin = np.isfinite(v) & (v != 0)
    _, e = np.frexp(v[fin])
    ulp = np.ldexp(1.0, np.maximum(e, -125) - 8)
    q = v[fin] / ulp
    out[fin] = np.sign(q) * np.floor(np.abs(q) + 0.5) * ulp
    return out


def _router_w_transposed(x_bits, router_w):
    w = np.asarray(router_w, np.float64)
    l64 = M.bf16_bits_to_f64(x_bits) @ w.reshape(w.shape[1], w.shape[0])
    return l64, l64.astype(np.float32)


def _bias_ignored(l32, bias):
    return np.asarray(l32, dtype=np.float32).copy()


def _route_nan_first(l32, k):
    l = np.asarray(l32, np.float32)
    return ORIG["route"](np.where(np.isnan(l), np.float32(np.inf), l), k)


ORIG = {n: getattr(M, n) for n in ("route", "batch_union", "moe_ffn_combine")}

MUTATIONS = {
    "nibble order swapped": ("unpack_int4", _swap_nibbles),
    "offset-8 codes instead of two's complement": ("unpack_int4", _offset_codes),
    "scale group index transposed": ("dequant", _interleaved_scales),
    "group size ignored (32 codes per scale)": ("dequant", _scale_per_32_codes),
    "int8 codes read unsigned": ("unpack_int8", _int8_unsigned),
    "ties to the highest index": ("route", _route_high_index_ties),
    "weights not renormalised": ("route", _route_not_renormalised),
    "union not stable": ("batch_union", _union_unstable),
    "h not rounded to bf16": ("expert_ffn_tokens", _ffn_no_h_round),
    "gate and up swapped": ("expert_ffn_tokens", _ffn_gate_up_swapped),
    "shared expert dropped": ("moe_ffn_combine", _combine_drop("shared")),
    "residual dropped": ("moe_ffn_combine", _combine_drop("residual")),
    "routing weights dropped": ("moe_ffn_combine", _combine_drop("weights")),
    "rms norm without sqrt": ("rms_norm", _rms_no_sqrt),
    "silu replaced by sigmoid": ("silu", _silu_as_sigmoid),
    "bf16 rounding wrong": ("round_bf16", _round_via_fp32),
    "bf16 ties away from zero": ("round_bf16", _round_ties_away),
    "router W_r read transposed": ("router_logits", _router_w_transposed),
    "bias ignored": ("add_bias", _bias_ignored),
    "NaN ranked first": ("route", _route_nan_first),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name, monkeypatch):
    fn, repl = MUTATIONS[name]
    monkeypatch.setattr(M, fn, repl)
    monkeypatch.setattr(oracle, fn, repl)
    assert _some_pin_fails(), f"no pin caught: {name}"


def test_pins_pass_unmutated():
    assert not _some_pin_fails()
