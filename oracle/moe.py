"""CPU oracle of the routed-expert MoE step (Route -> Union -> int4 SwiGLU -> combine).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  The product path (the CUDA library and its binding) never calls it and
shares no code with it.

Plain, slow and obviously correct: numpy in float64, one step per function, in
the order of the per-token path described on the Colibri README page
("Come funziona", "Il percorso di ogni token": Route, then Union, then the
expert matmuls) and in the getting-started guide ("トークンごとの処理経路":
1. Route, 2. Union).  The pages fix that routing is per token and per layer,
that positions of a batch read each unique expert once (README, "Mai aspettare
il disco due volte": batch-union), that routed experts live in an int4
container (README, "L'idea") and that where an expert is placed never changes
the router's decisions or the weights' precision (README, introduction and
"Il percorso di ogni token").  They give no formula; the numerics below are the
layer specification this library implements, and every place where it is a
reading rather than a statement is marked READING.

Parity pins live in ``tests/test_oracle_pins.py``; every function here is
pinned there.  ``oracle/c/moe_ref.c`` states the same layer again in plain C
by other means, and ``tests/test_oracle_c.py`` checks the two against each
other.
"""
from __future__ import annotations

import numpy as np

# --------------------------------------------------------------------------
# number formats
# --------------------------------------------------------------------------

BF16_MAX = float.fromhex("0x1.fe00000000000p+127")  # (2 - 2^-7) * 2^127


def fp16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """IEEE binary16 bit patterns -> float64 (exact)."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns -> float64 (exact): the top half of a binary32."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def round_bf16(v: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value (ties to even).

    bfloat16 keeps an 8-bit significand and binary32's exponent range, so a
    value in [2^(e-1), 2^e) is rounded to a multiple of 2^(e-8); below the
    smallest normal (2^-126) the spacing stays 2^-133.  Rounding is done once,
    straight from float64 (no intermediate binary32 rounding).  Magnitudes that
    round above the largest finite bfloat16 become infinities.
    Returns float64 arrays holding the bfloat16 values."""
    v = np.asarray(v, dtype=np.float64)
    out = np.array(v, copy=True)
    fin = np.isfinite(v) & (v != 0)
    _, e = np.frexp(v[fin])                      # v = m * 2^e, 0.5 <= |m| < 1
    e = np.maximum(e, -125)
    ulp = np.ldexp(1.0, e - 8)
    r = np.rint(v[fin] / ulp) * ulp              # np.rint: round half to even
    r[np.abs(r) > BF16_MAX] = np.copysign(np.inf, r[np.abs(r) > BF16_MAX])
    out[fin] = r
    return out


def f64_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """float64 -> bfloat16 bit patterns (round to nearest even, via round_bf16)."""
    r = round_bf16(v).astype(np.float32)         # exact: r has <= 8 significant bits
    return (r.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


# --------------------------------------------------------------------------
# C1: the int4 group-quantised container
# --------------------------------------------------------------------------

def unpack_int4(q_bytes: np.ndarray) -> np.ndarray:
    """Packed codes uint8 [rows, K/2] -> signed codes int8 [rows, K].

    READING (the pages say only "int4 container"; the layout is this library's):
    element c of a row sits in byte c // 2, in the low nibble when c is even
    and in the high nibble when c is odd; a nibble n is the two's-complement
    code n - 16 * (n >= 8), so codes span [-8, 7]."""
    b = np.asarray(q_bytes, dtype=np.uint8)
    nib = np.empty(b.shape[:-1] + (b.shape[-1] * 2,), dtype=np.int16)
    nib[..., 0::2] = b & 0x0F
    nib[..., 1::2] = b >> 4
    return (nib - 16 * (nib >= 8)).astype(np.int8)


def unpack_int8(q_bytes: np.ndarray) -> np.ndarray:
    """int8 container: codes uint8 [rows, K] -> signed codes int8 [rows, K].

    READING (the README requires the MTP head to be int8, "Decodifica
    speculativa, onestamente" and "2. Scarica il modello", but gives no
    layout): the int4 container with one byte per code, element c of a row
    in byte c, read as two's complement, so codes span [-128, 127]."""
    return np.asarray(q_bytes, dtype=np.uint8).view(np.int8).copy()


def dequant(q_bytes: np.ndarray, s_bits: np.ndarray, group: int = 32, bits: int = 4) -> np.ndarray:
    """Weights W[r, c] = code[r, c] * scale[r, c // group]   (float64, exact).

    Scales are fp16 [rows, K/group], one per group of ``group`` consecutive
    elements along K (the row).  ``bits`` selects the int4 (4) or int8 (8)
    code container."""
    q = (unpack_int4 if bits == 4 else unpack_int8)(q_bytes).astype(np.float64)
    s = fp16_bits_to_f64(s_bits)
    rows, k = q.shape
    assert s.shape == (rows, k // group)
    return (q.reshape(rows, k // group, group) * s[:, :, None]).reshape(rows, k)


# --------------------------------------------------------------------------
# C2/C3: router logits and bias
# --------------------------------------------------------------------------

def router_logits(x_bits: np.ndarray, router_w: np.ndarray):
    """l[t, e] = sum_h x[t, h] * W_r[e, h].

    x is bf16 [T, H], W_r fp32 [E, H].  Returns (float64 logits, the same
    rounded once to fp32)."""
    x = bf16_bits_to_f64(x_bits)
    l64 = x @ np.asarray(router_w, dtype=np.float64).T
    return l64, l64.astype(np.float32)


def add_bias(l32: np.ndarray, bias: np.ndarray | None) -> np.ndarray:
    """l'[t, e] = fp32(l[t, e] + bias[e]): one IEEE binary32 addition.

    READING: the additive per-expert bias enters both the selection and the
    weights."""
    l32 = np.asarray(l32, dtype=np.float32)
    if bias is None:
        return l32.copy()
    return (l32 + np.asarray(bias, dtype=np.float32)[None, :]).astype(np.float32)


# --------------------------------------------------------------------------
# C4/C5: Route (top-k with lowest-index ties, renormalised softmax weights)
# --------------------------------------------------------------------------

ST_NONFINITE = 1


def route(l32: np.ndarray, k: int):
    """Top-k selection and renormalised softmax weights, per token.

    Selection: the k largest logits under the total order
    (value descending, expert index ascending); slot j holds the j-th in that
    order.  A NaN logit ranks as -inf.  -0.0 and +0.0 tie.
    Weights: softmax over all E experts restricted to the selected k and
    renormalised, i.e. w_j = exp(l_j - l_max) / sum_{i in sel} exp(l_i - l_max)
    (the full softmax's denominator cancels), in float64.
    Returns (ids int32 [T,k], weights float64 [T,k], flags int [T]) where
    flags has ST_NONFINITE set when a logit is NaN or +inf or a selected
    logit is -inf (the weights are then not meaningful)."""
    l = np.asarray(l32, dtype=np.float32).astype(np.float64)
    T, E = l.shape
    key = np.where(np.isnan(l), -np.inf, l)
    idx = np.broadcast_to(np.arange(E), (T, E))
    # lexsort sorts by the last key first: primary = -value, secondary = index
    order = np.lexsort((idx, -key), axis=1)
    ids = order[:, :k].astype(np.int32)
    sel = np.take_along_axis(key, order[:, :k], axis=1)
    flags = np.zeros(T, dtype=np.int64)
    bad = np.isnan(l).any(1) | np.isposinf(l).any(1) | np.isneginf(sel).any(1)
    flags[bad] |= ST_NONFINITE
    with np.errstate(invalid="ignore", over="ignore"):
        e = np.exp(sel - sel[:, :1])
        w = e / e.sum(axis=1, keepdims=True)
    return ids, w, flags


# --------------------------------------------------------------------------
# C6: Union (batch-union of the selected experts)
# --------------------------------------------------------------------------

def batch_union(ids: np.ndarray, n_experts: int):
    """Dedupe the experts a batch selected and group its (token, slot) pairs.

    Pairs are numbered p = t*k + j.  Returns
      unique   int32 [U]   experts selected by at least one token, ascending;
      seg_off  int32 [U+1] seg_off[u]..seg_off[u+1] indexes perm for unique[u];
      perm     int32 [T*k] pairs ordered by (expert, p)  (stable by pair index,
                           hence by token, since a token never picks an
                           expert twice);
      pair_pos int32 [T*k] inverse of perm: pair p sits at perm[pair_pos[p]]."""
    flat = np.asarray(ids, dtype=np.int64).reshape(-1)
    assert flat.size == 0 or (flat.min() >= 0 and flat.max() < n_experts)
    perm = np.argsort(flat, kind="stable").astype(np.int32)
    unique, counts = np.unique(flat, return_counts=True)
    seg_off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    pair_pos = np.empty_like(perm)
    pair_pos[perm] = np.arange(flat.size, dtype=np.int32)
    return unique.astype(np.int32), seg_off, perm, pair_pos


# --------------------------------------------------------------------------
# C7/C8: expert SwiGLU FFN and routing-weighted combine
# --------------------------------------------------------------------------

def silu(g: np.ndarray) -> np.ndarray:
    """SiLU(g) = g / (1 + exp(-g)), float64."""
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g))


class ExpertWeights:
    """Access to expert e's dequantised matrices (float64), computed on demand.

    ``get_codes(kind, e)`` / ``get_scales(kind, e)`` return one expert's packed
    codes and fp16 scale bits for kind 'gate', 'up' or 'down'.  A small cache
    keeps the most recently dequantised matrices (``cache`` entries)."""

    def __init__(self, get_codes, get_scales, group: int = 32, cache: int = 0, bits: int = 4):
        self._c, self._s, self.group, self.bits = get_codes, get_scales, group, bits
        self._cache, self._cap = {}, cache

    def matrix(self, kind: str, e: int) -> np.ndarray:
        key = (kind, e)
        if key in self._cache:
            return self._cache[key]
        m = dequant(self._c(kind, e), self._s(kind, e), self.group, self.bits)
        if self._cap:
            if len(self._cache) >= self._cap:
                self._cache.pop(next(iter(self._cache)))
            self._cache[key] = m
        return m

    @staticmethod
    def from_synth(inputs, cache: int = 0) -> "ExpertWeights":
        """Adapter for ``synth.LayerInputs`` (regenerates one expert at a time)."""
        import synth
        qk = {"gate": synth.GATE_Q, "up": synth.UP_Q, "down": synth.DOWN_Q}
        sk = {"gate": synth.GATE_S, "up": synth.UP_S, "down": synth.DOWN_S}
        return ExpertWeights(lambda k, e: inputs.expert_codes(qk[k], e),
                             lambda k, e: inputs.expert_scales(sk[k], e),
                             inputs.shape.group, cache, inputs.shape.bits)

    @staticmethod
    def from_arrays(arrays: dict, group: int = 32, bits: int = 4) -> "ExpertWeights":
        """arrays: {'gate': (codes, scales), 'up': (...), 'down': (...)} with a
        leading expert axis."""
        return ExpertWeights(lambda k, e: arrays[k][0][e], lambda k, e: arrays[k][1][e], group, bits=bits)


def expert_ffn_tokens(W: ExpertWeights, e: int, x64: np.ndarray) -> np.ndarray:
    """y = W_down[e] . h with h = bf16(silu(W_gate[e] . x) * (W_up[e] . x)).

    x64: float64 [n, H] (bf16 values).  Gate/up are [I, H], down is [H, I].
    READING: h is rounded to bf16 (the tensor-core forms of the layer take a
    bf16 operand); everything else is float64.  Returns float64 [n, H]."""
    g = x64 @ W.matrix("gate", e).T
    u = x64 @ W.matrix("up", e).T
    h = round_bf16(silu(g) * u)
    return h @ W.matrix("down", e).T


def moe_ffn_combine(W: ExpertWeights, x_bits: np.ndarray, ids: np.ndarray, w: np.ndarray,
                    n_experts: int, n_shared: int, residual_bits: np.ndarray | None = None,
                    return_f64: bool = False):
    """out[t] = bf16( sum_j w[t,j] * y_{ids[t,j]}(x_t) + sum_s y_{E+s}(x_t) + residual[t] ).

    Walks the batch-union: each unique expert runs once over the tokens that
    selected it (README, "Mai aspettare il disco due volte": batch-union), then
    every token gathers its k routed outputs with their routing weights plus
    the shared experts' outputs (weight 1.0) and its residual; the sum is
    float64 and rounded once to bf16.  Returns bf16 bits [T, H] (and the
    float64 sum when ``return_f64``)."""
    x = bf16_bits_to_f64(x_bits)
    T, H = x.shape
    k = ids.shape[1]
    unique, seg_off, perm, _ = batch_union(ids, n_experts)
    acc = np.zeros((T, H), dtype=np.float64)
    for u, e in enumerate(unique):
        pairs = perm[seg_off[u]:seg_off[u + 1]]
        toks, slots = pairs // k, pairs % k
        y = expert_ffn_tokens(W, int(e), x[toks])
        acc[toks] += np.asarray(w, dtype=np.float64)[toks, slots][:, None] * y
    for s in range(n_shared):
        acc += expert_ffn_tokens(W, n_experts + s, x)
    if residual_bits is not None:
        acc += bf16_bits_to_f64(residual_bits)
    out = f64_to_bf16_bits(acc)
    return (out, acc) if return_f64 else out


# --------------------------------------------------------------------------
# the layer and the stack
# --------------------------------------------------------------------------

RMS_EPS = 1e-6


def rms_norm(h_bits: np.ndarray) -> np.ndarray:
    """n = bf16( h / sqrt(mean(h^2) + 1e-6) ), per token, float64 inside.

    READING: the pages and the layer statement name no normalisation; a
    weightless pre-norm is this library's reading for the 16-layer stack,
    whose literal form (h + MoE(h) carried in bf16) overflows bf16 within a
    few layers with the specified weight distributions."""
    h = bf16_bits_to_f64(h_bits)
    r = 1.0 / np.sqrt(np.mean(h * h, axis=1, keepdims=True) + RMS_EPS)
    return f64_to_bf16_bits(h * r)


def moe_layer(W: ExpertWeights, x_bits: np.ndarray, n_experts: int, top_k: int, n_shared: int,
              router_w: np.ndarray | None = None, bias: np.ndarray | None = None,
              logits_in: np.ndarray | None = None, residual_bits: np.ndarray | None = None,
              route_logits: np.ndarray | None = None):
    """One routed-expert MoE layer: logits -> Route -> Union -> FFN -> combine.

    ``logits_in`` (fp32 [T, E]) replaces x . W_r^T when given.  ``route_logits``
    lets a caller route from given fp32 logits (after the bias is added) while
    still returning the oracle's own logits for comparison.
    Returns dict with logits64, logits32, ids, w, flags, out (bf16 bits)."""
    if logits_in is not None:
        l32 = np.asarray(logits_in, dtype=np.float32)
        l64 = l32.astype(np.float64)
    else:
        l64, l32 = router_logits(x_bits, router_w)
    lb = add_bias(l32 if route_logits is None else route_logits, bias)
    ids, w, flags = route(lb, top_k)
    out = moe_ffn_combine(W, x_bits, ids, w, n_experts, n_shared, residual_bits)
    return {"logits64": l64, "logits32": l32, "ids": ids, "w": w, "flags": flags, "out": out}


def moe_stack(layers, h0_bits: np.ndarray, n_experts: int, top_k: int, n_shared: int):
    """h_{l+1} = bf16( h_l + MoE_l( rms_norm(h_l) ) ) for each layer l.

    ``layers`` is a list of (ExpertWeights, router_w, bias) per layer.
    Returns (final hidden bf16 bits, list of per-layer dicts)."""
    h = np.asarray(h0_bits, dtype=np.uint16)
    per = []
    for W, rw, bias in layers:
        n = rms_norm(h)
        r = moe_layer(W, n, n_experts, top_k, n_shared, router_w=rw, bias=bias, residual_bits=h)
        r["normed"] = n
        per.append(r)
        h = r["out"]
    return h, per
