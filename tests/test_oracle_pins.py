"""Pins of the CPU oracle to things other than itself.

Each test ties one oracle function to a hand-worked example (``tests/golden``),
a brute-force enumeration, a closed form, an invariant, or an independent
library routine, so that a dropped term, a wrong sign or index, or a transposed
operand anywhere in the oracle fails at least one of them.  CPU only.
"""
import itertools
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLD, name)) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]


# ---------------------------------------------------------------- formats

def test_unpack_roundtrip_all_code_pairs():
    """Pack every (even, odd) code pair with Python's two's-complement '&' and
    unpack with the oracle: the codes come back."""
    pairs = list(itertools.product(range(-8, 8), repeat=2))
    packed = np.array([[(lo & 0xF) | ((hi & 0xF) << 4) for lo, hi in pairs]], dtype=np.uint8)
    codes = oracle.unpack_int4(packed).reshape(-1, 2)
    assert codes.tolist() == [list(p) for p in pairs]
    assert sorted(set(packed[0].tolist())) == list(range(256))


def test_dequant_hand_worked():
    rows = _golden("dequant_hand.txt")
    for ln in rows:
        f = [p.strip() for p in ln.split("|")]
        if f[0] == "ROW":
            b = [int(v, 16) for v in f[1].split()] + [0] * 28
            s = [int(v, 16) for v in f[2].split()]
            want = [float(v) for v in f[3].split()] + [0.0] * 56
            W = oracle.dequant(np.array([b], np.uint8), np.array([s], np.uint16), 32)
            assert W.shape == (1, 64)
            assert W[0].tolist() == want
            continue
        byte, sb = int(f[0], 16), int(f[1], 16)
        row = np.array([[byte] * 16], np.uint8)
        W = oracle.dequant(row, np.array([[sb]], np.uint16), 32)
        assert W[0, 0] == float(f[2]) and W[0, 1] == float(f[3])
        assert W[0, 30] == float(f[2]) and W[0, 31] == float(f[3])


def test_unpack_int8_every_byte():
    """Every byte value decodes to its two's-complement code (Python's own
    signed conversion, not numpy's)."""
    b = np.arange(256, dtype=np.uint8).reshape(1, 256)
    want = [int.from_bytes(bytes([v]), "little", signed=True) for v in range(256)]
    assert oracle.unpack_int8(b)[0].tolist() == want


def test_dequant_int8_hand_worked():
    for ln in _golden("dequant_int8_hand.txt"):
        f = [p.strip() for p in ln.split("|")]
        byte, sb, want = int(f[0], 16), int(f[1], 16), float(f[2])
        W = oracle.dequant(np.array([[byte] * 32], np.uint8), np.array([[sb]], np.uint16), 32, bits=8)
        assert W.shape == (1, 32)
        assert W[0].tolist() == [want] * 32


def test_dequant_int8_group_index_and_rows():
    _check_group_index(32, bits=8)
    _check_group_index(64, bits=8)


def test_dequant_group_index_and_rows():
    _check_group_index(32)


def test_dequant_gs64_group_index_and_rows():
    """Group 64 is the gs64 container (Colibri README, "2. Scarica il modello")."""
    _check_group_index(64)


def _check_group_index(group, bits=4):
    """Scale (r, c // group) multiplies element (r, c): each scale set to a
    power of two tagging its (row, group) is recovered from a code-1 matrix."""
    rows, K = 3, 256
    ng = K // group
    q = np.full((rows, K // 2), 0x11, np.uint8) if bits == 4 else np.full((rows, K), 0x01, np.uint8)  # codes = +1
    s = np.zeros((rows, ng), np.float16)
    for r in range(rows):
        for g in range(ng):
            s[r, g] = 2.0 ** -(r * ng + g)
    W = oracle.dequant(q, s.view(np.uint16), group, bits)
    for r in range(rows):
        for c in range(K):
            assert W[r, c] == 2.0 ** -(r * ng + c // group)


def test_dequant_gs64_is_gs32_with_paired_scales():
    """A group-64 container equals the group-32 container whose two scales of
    every 64-wide span are both that span's scale (seeded codes and scales)."""
    rng = np.random.default_rng(64)
    rows, K = 5, 512
    q = rng.integers(0, 256, (rows, K // 2), dtype=np.uint8)
    s64 = rng.uniform(0.005, 0.02, (rows, K // 64)).astype(np.float16)
    s32 = np.repeat(s64, 2, axis=1)
    W64 = oracle.dequant(q, s64.view(np.uint16), 64)
    W32 = oracle.dequant(q, s32.view(np.uint16), 32)
    assert np.array_equal(W64, W32)
    codes = oracle.unpack_int4(q).astype(np.float64)
    assert np.array_equal(W64, codes * np.repeat(s64.astype(np.float64), 64, axis=1))


def test_round_bf16_matches_torch_on_fp32_inputs():
    rng = np.random.default_rng(1)
    v = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(37.0),
        # exact ties: bf16 value +/- half an ulp
        (np.arange(1, 2000, dtype=np.float32) * np.float32(2 ** -7) + np.float32(2 ** -8) + 1).astype(np.float32),
        np.array([3.3895313e38, 3.4e38, -3.4e38, 1e-40, -1e-41, 0.0, -0.0], np.float32),
    ]).astype(np.float32)
    want = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.round_bf16(v.astype(np.float64))
    assert np.array_equal(got, want, equal_nan=True)
    bits = oracle.f64_to_bf16_bits(v.astype(np.float64))
    assert np.array_equal(bits, torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))


def test_round_bf16_rounds_once_from_double():
    # 1 + 2^-8 + 2^-40: above the tie, so it rounds up to 1 + 2^-7.  Rounding to
    # fp32 first would land on the tie 1 + 2^-8 and then go down to 1.0.
    v = 1.0 + 2.0 ** -8 + 2.0 ** -40
    assert oracle.round_bf16(np.array([v]))[0] == 1.0 + 2.0 ** -7
    assert oracle.round_bf16(np.array([1.0 + 2.0 ** -8]))[0] == 1.0       # tie -> even
    assert oracle.round_bf16(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 1.0 + 2.0 ** -6  # tie -> even (up)


# ---------------------------------------------------------------- logits and bias

def test_router_logits_exact_integer_case():
    """Small integer x and W_r: dot products are exact; compare with Python ints."""
    rng = np.random.default_rng(2)
    T, E, H = 3, 5, 64
    xi = rng.integers(-4, 5, size=(T, H))
    wi = rng.integers(-3, 4, size=(E, H))
    x_bits = synth.f32_to_bf16_bits(xi.astype(np.float32))
    l64, l32 = oracle.router_logits(x_bits, wi.astype(np.float32))
    for t in range(T):
        for e in range(E):
            assert l64[t, e] == sum(int(xi[t, h]) * int(wi[e, h]) for h in range(H))
    # operand orientation: a one-hot token reads one column of W_r^T
    x1 = np.zeros((1, H), np.float32)
    x1[0, 7] = 1.0
    l64, _ = oracle.router_logits(synth.f32_to_bf16_bits(x1), wi.astype(np.float32))
    assert l64[0].tolist() == wi[:, 7].astype(float).tolist()


def test_add_bias_is_one_fp32_add():
    import struct
    rng = np.random.default_rng(3)
    l = rng.standard_normal((4, 9)).astype(np.float32)
    b = rng.standard_normal(9).astype(np.float32)
    got = oracle.add_bias(l, b)
    for t in range(4):
        for e in range(9):
            exact = float(l[t, e]) + float(b[e])          # exact in double
            want = struct.unpack("f", struct.pack("f", exact))[0]
            assert got[t, e] == np.float32(want)
    assert np.array_equal(oracle.add_bias(l, None), l)


# ---------------------------------------------------------------- route

def _brute_topk(l, k):
    """The unique k-subset S with l_i > l_j or (l_i == l_j and i < j) for all i in S, j not in S."""
    E = len(l)
    found = []
    for S in itertools.combinations(range(E), k):
        out = [j for j in range(E) if j not in S]
        if all(l[i] > l[j] or (l[i] == l[j] and i < j) for i in S for j in out):
            found.append(S)
    assert len(found) == 1
    return set(found[0])


def test_route_matches_brute_force_on_tie_dense_logits():
    rng = np.random.default_rng(4)
    for trial in range(1500):
        E = int(rng.integers(2, 9))
        k = int(rng.integers(1, E + 1))
        l = rng.integers(0, 4, size=(1, E)).astype(np.float32)
        ids, w, flags = oracle.route(l, k)
        assert set(ids[0].tolist()) == _brute_topk(l[0].tolist(), k)
        # slot order: value descending, index ascending
        keys = [(-l[0, e], e) for e in ids[0]]
        assert keys == sorted(keys)
        assert flags[0] == 0


def test_route_weights_special_cases_and_softmax_identity():
    rng = np.random.default_rng(5)
    # k = 1 -> weight exactly 1
    ids, w, _ = oracle.route(rng.standard_normal((7, 16)).astype(np.float32), 1)
    assert np.all(w == 1.0)
    # all logits equal -> ids 0..k-1, weights 1/k
    ids, w, _ = oracle.route(np.full((2, 10), 0.75, np.float32), 4)
    assert ids.tolist() == [[0, 1, 2, 3]] * 2 and np.all(w == 0.25)
    # k = 2: w = (sigmoid(l1 - l2), sigmoid(l2 - l1))
    l = rng.standard_normal((50, 12)).astype(np.float32) * 3
    ids, w, _ = oracle.route(l, 2)
    l1 = np.take_along_axis(l, ids, 1).astype(np.float64)
    assert np.allclose(w[:, 0], scipy.special.expit(l1[:, 0] - l1[:, 1]), rtol=0, atol=1e-15)
    # general k: renormalised full softmax (scipy), same selection
    for k in (3, 8):
        ids, w, _ = oracle.route(l, k)
        p = scipy.special.softmax(l.astype(np.float64), axis=1)
        ps = np.take_along_axis(p, ids, 1)
        assert np.allclose(w, ps / ps.sum(1, keepdims=True), rtol=1e-13, atol=0)
        assert np.allclose(w.sum(1), 1.0, rtol=0, atol=1e-12)
        assert np.all(np.diff(w, axis=1) <= 0)


def test_route_hand_worked():
    for ln in _golden("route_hand.txt"):
        _, ls, ks, idss, ws = [p.strip() for p in ln.split("|")]
        l = np.array([[float(v) for v in ls.split()]], np.float32)
        ids, w, flags = oracle.route(l, int(ks))
        assert ids[0].tolist() == [int(v) for v in idss.split()]
        assert np.allclose(w[0], [float(v) for v in ws.split()], rtol=0, atol=2e-16)
        assert flags[0] == 0


def test_route_nonfinite_flags():
    l = np.array([[0.0, np.nan, 1.0, -np.inf],
                  [0.0, 2.0, np.inf, 1.0],
                  [-np.inf, -np.inf, 1.0, -np.inf],
                  [-np.inf, 3.0, 1.0, 2.0]], np.float32)
    ids, w, flags = oracle.route(l, 2)
    assert ids[0].tolist() == [2, 0]          # NaN ranks as -inf
    assert flags.tolist() == [1, 1, 1, 0]     # NaN; +inf; a selected -inf; clean
    assert ids[2].tolist() == [2, 0]          # -inf ties broken by index


# ---------------------------------------------------------------- union

def _brute_union(flat, E):
    unique, seg_off, perm = [], [0], []
    for e in range(E):
        members = [p for p in range(len(flat)) if flat[p] == e]
        if members:
            unique.append(e)
            perm.extend(members)
            seg_off.append(len(perm))
    return unique, seg_off, perm


@pytest.mark.parametrize("T,E,k", [(1, 16, 2), (4, 16, 2), (9, 5, 5), (33, 40, 3), (64, 256, 8), (0, 8, 2)])
def test_batch_union_brute_force_and_invariants(T, E, k):
    rng = np.random.default_rng(T * 100 + E)
    ids = np.array([rng.choice(E, size=k, replace=False) for _ in range(T)], np.int32).reshape(T, k)
    unique, seg_off, perm, pair_pos = oracle.batch_union(ids, E)
    bu, bs, bp = _brute_union(ids.reshape(-1).tolist(), E)
    assert unique.tolist() == bu and seg_off.tolist() == bs and perm.tolist() == bp
    # invariants
    assert np.all(np.diff(unique) > 0)
    assert seg_off[0] == 0 and seg_off[-1] == T * k and np.all(np.diff(seg_off) > 0)
    assert np.array_equal(perm[pair_pos], np.arange(T * k))
    tok_count = np.zeros(T, int)
    for u in range(len(unique)):
        toks = perm[seg_off[u]:seg_off[u + 1]] // max(k, 1)
        assert len(set(toks.tolist())) == len(toks)      # a token at most once per segment
        assert np.all(np.diff(toks) > 0)                  # ascending token order
        tok_count[toks] += 1
    assert np.all(tok_count == k)


# ---------------------------------------------------------------- FFN and combine

def test_silu_matches_library():
    g = np.linspace(-30, 30, 2001)
    assert np.allclose(oracle.silu(g), g * scipy.special.expit(g), rtol=1e-14, atol=1e-300)
    assert oracle.silu(np.array([0.0]))[0] == 0.0


def _rand_layer(rng, H, I, E, S, zero_routed=False, bits=4):
    n = E + S
    arr = {}
    for kind, (r, K) in {"gate": (I, H), "up": (I, H), "down": (H, I)}.items():
        c = rng.integers(0, 256, size=(n, r, K * bits // 8), dtype=np.uint8)
        if zero_routed:
            c[:E] = 0
        s = rng.uniform(0.005, 0.02, size=(n, r, K // 32)).astype(np.float16).view(np.uint16)
        arr[kind] = (c, s)
    return arr


def _py_dequant(codes, scales, bits=4):
    """Pure-Python dequant from the container definition (independent loops)."""
    rows, kb = codes.shape
    K = kb * 8 // bits
    out = [[0.0] * K for _ in range(rows)]
    for r in range(rows):
        for c in range(K):
            if bits == 4:
                byte = int(codes[r, c // 2])
                nib = (byte >> 4) if (c % 2) else (byte & 15)
                code = nib - 16 if nib > 7 else nib
            else:
                byte = int(codes[r, c])
                code = byte - 256 if byte > 127 else byte
            out[r][c] = code * float(np.uint16(scales[r, c // 32]).view(np.float16))
    return out


def _py_dense_swiglu(x, Wg, Wu, Wd):
    """Dense SwiGLU FFN with plain Python loops; h rounded to bf16."""
    I, H = len(Wg), len(Wg[0])
    g = [sum(Wg[i][c] * x[c] for c in range(H)) for i in range(I)]
    u = [sum(Wu[i][c] * x[c] for c in range(H)) for i in range(I)]
    h = [gi / (1.0 + math.exp(-gi)) * ui for gi, ui in zip(g, u)]
    h = [float(torch.tensor(v, dtype=torch.float64).to(torch.bfloat16).to(torch.float64)) if abs(v) < 1e30 else v
         for v in h]
    return [sum(Wd[r][i] * h[i] for i in range(I)) for r in range(H)]


def test_dense_identity_one_expert():
    """E=1, k=1, S=0: the layer equals a dense SwiGLU FFN (Python loops)."""
    _dense_identity(bits=4)


def test_dense_identity_one_expert_int8():
    _dense_identity(bits=8)


def _dense_identity(bits):
    rng = np.random.default_rng(6)
    H, I, T = 64, 32, 3
    arr = _rand_layer(rng, H, I, 1, 0, bits=bits)
    W = oracle.ExpertWeights.from_arrays(arr, bits=bits)
    x_bits = synth.normal_bf16(9, 0, 1, (T, H))
    ids = np.zeros((T, 1), np.int32)
    out, acc = oracle.moe_ffn_combine(W, x_bits, ids, np.ones((T, 1)), 1, 0, return_f64=True)
    Wg, Wu, Wd = (_py_dequant(*(a[0] for a in arr[k]), bits=bits) for k in ("gate", "up", "down"))
    for t in range(T):
        x = oracle.bf16_bits_to_f64(x_bits[t]).tolist()
        ref = _py_dense_swiglu(x, Wg, Wu, Wd)
        assert np.allclose(acc[t], ref, rtol=1e-12, atol=1e-12 * max(map(abs, ref)))
        assert oracle.bf16_bits_to_f64(out[t]).tolist() == oracle.round_bf16(np.array(ref)).tolist()


def test_shared_expert_alone_is_dense():
    """Routed experts with zero codes: the output is the shared expert's dense FFN."""
    rng = np.random.default_rng(7)
    H, I, E, T = 64, 32, 4, 2
    arr = _rand_layer(rng, H, I, E, 1, zero_routed=True)
    W = oracle.ExpertWeights.from_arrays(arr)
    x_bits = synth.normal_bf16(10, 0, 1, (T, H))
    ids, w, _ = oracle.route(rng.standard_normal((T, E)).astype(np.float32), 2)
    _, acc = oracle.moe_ffn_combine(W, x_bits, ids, w, E, 1, return_f64=True)
    Wg, Wu, Wd = (_py_dequant(*(a[E] for a in arr[k])) for k in ("gate", "up", "down"))
    for t in range(T):
        ref = _py_dense_swiglu(oracle.bf16_bits_to_f64(x_bits[t]).tolist(), Wg, Wu, Wd)
        assert np.allclose(acc[t], ref, rtol=1e-12, atol=1e-12 * max(map(abs, ref)))


def test_combine_is_routing_weighted_sum_of_dense_experts():
    """E=3, k=2: out = w0 * dense_{id0}(x) + w1 * dense_{id1}(x) + residual."""
    rng = np.random.default_rng(8)
    H, I, E, T = 32, 32, 3, 3
    arr = _rand_layer(rng, H, I, E, 0)
    W = oracle.ExpertWeights.from_arrays(arr)
    x_bits = synth.normal_bf16(11, 0, 1, (T, H))
    res_bits = synth.normal_bf16(12, 0, 1, (T, H))
    ids, w, _ = oracle.route(rng.standard_normal((T, E)).astype(np.float32), 2)
    _, acc = oracle.moe_ffn_combine(W, x_bits, ids, w, E, 0, residual_bits=res_bits, return_f64=True)
    dense = [[_py_dequant(*(a[e] for a in arr[k])) for k in ("gate", "up", "down")] for e in range(E)]
    for t in range(T):
        x = oracle.bf16_bits_to_f64(x_bits[t]).tolist()
        ref = np.array(oracle.bf16_bits_to_f64(res_bits[t]))
        for j in range(2):
            ref = ref + w[t, j] * np.array(_py_dense_swiglu(x, *dense[ids[t, j]]))
        assert np.allclose(acc[t], ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_ffn_one_code_hand_worked():
    g = {ln.split()[0]: ln for ln in _golden("ffn_one_code.txt")}
    H = I = 32
    arr = {k: (np.zeros((1, r, K // 2), np.uint8), np.zeros((1, r, K // 32), np.uint16))
           for k, (r, K) in {"gate": (I, H), "up": (I, H), "down": (H, I)}.items()}
    for kind in ("gate", "up", "down"):
        _, r, c, code, sbits = g[kind].split()
        r, c, code = int(r), int(c), int(code)
        arr[kind][0][0, r, c // 2] |= (code & 0xF) << (4 * (c % 2))
        arr[kind][1][0, r, c // 32] = int(sbits, 16)
    W = oracle.ExpertWeights.from_arrays(arr)
    x = np.zeros((1, H), np.float32)
    x[0, 3] = 2.0
    out = oracle.moe_ffn_combine(W, synth.f32_to_bf16_bits(x), np.zeros((1, 1), np.int32),
                                 np.ones((1, 1)), 1, 0)
    want = np.zeros(H)
    _, r, v = g["out"].split()
    want[int(r)] = float(v)
    assert oracle.bf16_bits_to_f64(out[0]).tolist() == want.tolist()
    # the intermediate h of the worked example
    gg = x.astype(np.float64) @ W.matrix("gate", 0).T
    uu = x.astype(np.float64) @ W.matrix("up", 0).T
    h = oracle.round_bf16(oracle.silu(gg) * uu)
    _, r, v = g["h"].split()
    assert h[0, int(r)] == float(v) and np.count_nonzero(h) == 1


def test_zero_codes_give_residual_and_down_scale_doubles_output():
    rng = np.random.default_rng(9)
    H, I, E, S, T = 64, 32, 4, 1, 3
    arr = _rand_layer(rng, H, I, E, S)
    x_bits = synth.normal_bf16(13, 0, 1, (T, H))
    res = synth.normal_bf16(14, 0, 1, (T, H))
    ids, w, _ = oracle.route(rng.standard_normal((T, E)).astype(np.float32), 2)
    zero = {k: (np.zeros_like(v[0]), v[1]) for k, v in arr.items()}
    out = oracle.moe_ffn_combine(oracle.ExpertWeights.from_arrays(zero), x_bits, ids, w, E, S, residual_bits=res)
    assert np.array_equal(out, res)
    _, a1 = oracle.moe_ffn_combine(oracle.ExpertWeights.from_arrays(arr), x_bits, ids, w, E, S, return_f64=True)
    dbl = dict(arr)
    s2 = (arr["down"][1].view(np.float16).astype(np.float32) * 2).astype(np.float16).view(np.uint16)
    dbl["down"] = (arr["down"][0], s2)
    _, a2 = oracle.moe_ffn_combine(oracle.ExpertWeights.from_arrays(dbl), x_bits, ids, w, E, S, return_f64=True)
    assert np.array_equal(a2, 2 * a1)


def test_token_and_expert_permutation_and_batch_split():
    rng = np.random.default_rng(10)
    H, I, E, S, T, k = 64, 32, 6, 1, 5, 2
    arr = _rand_layer(rng, H, I, E, S)
    W = oracle.ExpertWeights.from_arrays(arr)
    x_bits = synth.normal_bf16(15, 0, 1, (T, H))
    rw = rng.standard_normal((E, H)).astype(np.float32) * 0.1
    base = oracle.moe_layer(W, x_bits, E, k, S, router_w=rw)
    # token permutation permutes rows
    p = rng.permutation(T)
    r = oracle.moe_layer(W, x_bits[p], E, k, S, router_w=rw)
    assert np.array_equal(r["out"], base["out"][p])
    # relabel experts consistently (weights and router rows): same output
    q = rng.permutation(E)          # new id of old expert e is q[e]
    inv = np.argsort(q)
    arr2 = {kk: (np.concatenate([v[0][inv], v[0][E:]]), np.concatenate([v[1][inv], v[1][E:]])) for kk, v in arr.items()}
    r2 = oracle.moe_layer(oracle.ExpertWeights.from_arrays(arr2), x_bits, E, k, S, router_w=rw[inv])
    assert np.array_equal(r2["out"], base["out"])
    # one token at a time gives the same result
    for t in range(T):
        rt = oracle.moe_layer(W, x_bits[t:t + 1], E, k, S, router_w=rw)
        assert np.array_equal(rt["out"][0], base["out"][t])


def test_rms_norm_matches_library():
    h = synth.normal_bf16(16, 0, 1, (5, 256))
    hf = torch.from_numpy(oracle.bf16_bits_to_f64(h))
    ref = torch.nn.functional.rms_norm(hf, (256,), eps=oracle.RMS_EPS)
    assert np.array_equal(oracle.bf16_bits_to_f64(oracle.rms_norm(h)), oracle.round_bf16(ref.numpy()))
    c = synth.f32_to_bf16_bits(np.full((1, 64), 3.0, np.float32))
    assert np.all(oracle.bf16_bits_to_f64(oracle.rms_norm(c)) == 1.0)


def test_stack_one_layer_is_residual_plus_normed_layer():
    rng = np.random.default_rng(11)
    H, I, E, S, T, k = 64, 32, 4, 1, 3, 2
    arr = _rand_layer(rng, H, I, E, S)
    W = oracle.ExpertWeights.from_arrays(arr)
    rw = rng.standard_normal((E, H)).astype(np.float32) * 0.1
    h0 = synth.normal_bf16(17, 0, 1, (T, H))
    hN, per = oracle.moe_stack([(W, rw, None)], h0, E, k, S)
    n = oracle.rms_norm(h0)
    r = oracle.moe_layer(W, n, E, k, S, router_w=rw)
    _, acc = oracle.moe_ffn_combine(W, n, r["ids"], r["w"], E, S, return_f64=True)
    want = oracle.f64_to_bf16_bits(acc + oracle.bf16_bits_to_f64(h0))
    assert np.array_equal(hN, want)
    assert np.array_equal(per[0]["ids"], r["ids"])
