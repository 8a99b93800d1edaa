"""The plain-C oracle (``oracle/c/moe_ref.c``): pinned like the numpy oracle, then
checked against it.

The C oracle states the same layer from the definitions (bit fields, a bit-level
bf16 rounding, selection passes, a counting sort, sequential double sums), so
agreement between the two on seeded layers ties each to the other through
independent means.  Both sides first pass the same pins: the hand-worked
fixtures under ``tests/golden``, brute-force top-k and union, library
conversions, and the dense SwiGLU identity.  CPU only (needs gcc).
"""
import itertools

import numpy as np
import pytest
import scipy.special
import torch

import oracle
import oracle.cref as cr
import synth
from tests.test_oracle_pins import (_brute_topk, _brute_union, _golden, _py_dense_swiglu, _py_dequant,
                                    _rand_layer)


# ---------------------------------------------------------------- formats

def test_decode_every_fp16_and_bf16_pattern():
    b = np.arange(65536, dtype=np.uint16)
    assert np.array_equal(cr.decode_fp16(b), b.view(np.float16).astype(np.float64), equal_nan=True)
    want = torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(cr.decode_bf16(b), want, equal_nan=True)


def test_round_bf16_matches_torch_on_fp32_inputs():
    rng = np.random.default_rng(21)
    v = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(37.0),
        (np.arange(1, 2000, dtype=np.float32) * np.float32(2 ** -7) + np.float32(2 ** -8) + 1).astype(np.float32),
        np.array([3.3895313e38, 3.4e38, -3.4e38, 1e-40, -1e-41, 0.0, -0.0, np.inf, -np.inf], np.float32),
        # bfloat16 subnormals and the ties between them
        (np.arange(-300, 300, dtype=np.float64) * 2.0 ** -134).astype(np.float32),
    ]).astype(np.float32)
    t = torch.from_numpy(v).to(torch.bfloat16)
    assert np.array_equal(cr.round_bf16(v.astype(np.float64)), t.to(torch.float64).numpy())
    assert np.array_equal(cr.f64_to_bf16_bits(v.astype(np.float64)), t.view(torch.int16).numpy().view(np.uint16))


def test_round_bf16_rounds_once_from_double():
    v = np.array([1.0 + 2.0 ** -8 + 2.0 ** -40, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8,
                  -(1.0 + 2.0 ** -8 + 2.0 ** -40), 2.0 ** -130 + 2.0 ** -134 + 2.0 ** -160])
    want = [1.0 + 2.0 ** -7, 1.0, 1.0 + 2.0 ** -6, -(1.0 + 2.0 ** -7), 2.0 ** -130 + 2.0 ** -133]
    assert cr.round_bf16(v).tolist() == want


def test_round_bf16_overflow_boundary():
    top = (2 - 2.0 ** -7) * 2.0 ** 127
    half_ulp = 2.0 ** 119
    got = cr.round_bf16(np.array([top, top + half_ulp * 0.999, top + half_ulp, -(top + 2 * half_ulp)]))
    assert got.tolist() == [top, top, np.inf, -np.inf]   # the tie rounds to even, i.e. 2^128


def test_dequant_hand_worked():
    for ln in _golden("dequant_hand.txt"):
        f = [p.strip() for p in ln.split("|")]
        if f[0] == "ROW":
            b = [int(v, 16) for v in f[1].split()] + [0] * 28
            s = [int(v, 16) for v in f[2].split()]
            want = [float(v) for v in f[3].split()] + [0.0] * 56
            assert cr.dequant(np.array([b], np.uint8), np.array([s], np.uint16), 32)[0].tolist() == want
            continue
        byte, sb = int(f[0], 16), int(f[1], 16)
        W = cr.dequant(np.array([[byte] * 16], np.uint8), np.array([[sb]], np.uint16), 32)
        assert W[0, 0] == float(f[2]) and W[0, 1] == float(f[3])
        assert W[0, 30] == float(f[2]) and W[0, 31] == float(f[3])
    for ln in _golden("dequant_int8_hand.txt"):
        f = [p.strip() for p in ln.split("|")]
        W = cr.dequant(np.array([[int(f[0], 16)] * 32], np.uint8), np.array([[int(f[1], 16)]], np.uint16), 32, 8)
        assert W[0].tolist() == [float(f[2])] * 32


@pytest.mark.parametrize("group,bits", [(32, 4), (64, 4), (32, 8), (64, 8)])
def test_dequant_group_index_and_rows(group, bits):
    rows, K = 3, 256
    ng = K // group
    q = np.full((rows, K // 2), 0x11, np.uint8) if bits == 4 else np.full((rows, K), 0x01, np.uint8)
    s = np.array([[2.0 ** -(r * ng + g) for g in range(ng)] for r in range(rows)], np.float16)
    W = cr.dequant(q, s.view(np.uint16), group, bits)
    for r in range(rows):
        assert W[r].tolist() == [2.0 ** -(r * ng + c // group) for c in range(K)]


def test_dequant_matches_python_loops_every_code():
    rng = np.random.default_rng(22)
    for bits in (4, 8):
        q = rng.integers(0, 256, size=(4, 64 * bits // 8), dtype=np.uint8)
        s = rng.uniform(0.005, 0.02, size=(4, 2)).astype(np.float16).view(np.uint16)
        assert cr.dequant(q, s, 32, bits).tolist() == _py_dequant(q, s, bits)


# ---------------------------------------------------------------- logits, route, union

def test_router_logits_exact_integer_case():
    rng = np.random.default_rng(23)
    T, E, H = 3, 5, 64
    xi, wi = rng.integers(-4, 5, size=(T, H)), rng.integers(-3, 4, size=(E, H))
    l64, l32 = cr.router_logits(synth.f32_to_bf16_bits(xi.astype(np.float32)), wi.astype(np.float32))
    assert l64.tolist() == (xi @ wi.T).astype(float).tolist()
    assert np.array_equal(l32, (xi @ wi.T).astype(np.float32))


def test_route_matches_brute_force_on_tie_dense_logits():
    rng = np.random.default_rng(24)
    for _ in range(1500):
        E = int(rng.integers(2, 9))
        k = int(rng.integers(1, E + 1))
        l = rng.integers(0, 4, size=(1, E)).astype(np.float32)
        ids, w, flags = cr.route(l, k)
        assert set(ids[0].tolist()) == _brute_topk(l[0].tolist(), k)
        keys = [(-l[0, e], e) for e in ids[0]]
        assert keys == sorted(keys) and flags[0] == 0


def test_route_hand_worked_and_softmax_identity():
    for ln in _golden("route_hand.txt"):
        _, ls, ks, idss, ws = [p.strip() for p in ln.split("|")]
        ids, w, flags = cr.route(np.array([[float(v) for v in ls.split()]], np.float32), int(ks))
        assert ids[0].tolist() == [int(v) for v in idss.split()]
        assert np.allclose(w[0], [float(v) for v in ws.split()], rtol=0, atol=2e-16) and flags[0] == 0
    l = np.random.default_rng(25).standard_normal((50, 12)).astype(np.float32) * 3
    for k in (1, 2, 3, 8):
        ids, w, _ = cr.route(l, k)
        p = np.take_along_axis(scipy.special.softmax(l.astype(np.float64), axis=1), ids, 1)
        assert np.allclose(w, p / p.sum(1, keepdims=True), rtol=1e-13, atol=0)


def test_route_bias_is_one_fp32_add_before_selection():
    rng = np.random.default_rng(26)
    l = rng.standard_normal((40, 16)).astype(np.float32)
    b = (rng.standard_normal(16) * 2).astype(np.float32)
    ids, w, f = cr.route(l, 4, bias=b)
    ids2, w2, f2 = cr.route((l + b[None, :]).astype(np.float32), 4)
    assert np.array_equal(ids, ids2) and np.array_equal(w, w2) and np.array_equal(f, f2)


def test_route_nonfinite_flags():
    l = np.array([[0.0, np.nan, 1.0, -np.inf],
                  [0.0, 2.0, np.inf, 1.0],
                  [-np.inf, -np.inf, 1.0, -np.inf],
                  [-np.inf, 3.0, 1.0, 2.0],
                  [np.nan, 0.5, 2.0, 1.0]], np.float32)
    ids, _, flags = cr.route(l, 2)
    assert ids[0].tolist() == [2, 0] and ids[2].tolist() == [2, 0]
    assert ids[4].tolist() == [2, 3]          # a NaN in slot 0's first candidate still ranks last
    assert flags.tolist() == [1, 1, 1, 0, 1]


@pytest.mark.parametrize("T,E,k", [(1, 16, 2), (4, 16, 2), (9, 5, 5), (33, 40, 3), (64, 256, 8), (0, 8, 2)])
def test_batch_union_brute_force_and_inverse(T, E, k):
    rng = np.random.default_rng(T * 7 + E)
    ids = np.array([rng.choice(E, size=k, replace=False) for _ in range(T)], np.int32).reshape(T, k)
    unique, seg_off, perm, pair_pos = cr.batch_union(ids, E)
    bu, bs, bp = _brute_union(ids.reshape(-1).tolist(), E)
    assert unique.tolist() == bu and seg_off.tolist() == bs and perm.tolist() == bp
    assert np.array_equal(perm[pair_pos], np.arange(T * k))


def test_union_rejects_out_of_range_ids():
    with pytest.raises(ValueError):
        cr.batch_union(np.array([[0, 8]], np.int32), 8)
    with pytest.raises(ValueError):
        cr.route(np.zeros((1, 4), np.float32), 5)


# ---------------------------------------------------------------- FFN, combine, layer

@pytest.mark.parametrize("bits", [4, 8])
def test_dense_identity_one_expert(bits):
    """E=1, k=1, S=0: the layer is a dense SwiGLU FFN (Python loops)."""
    rng = np.random.default_rng(27)
    H, I, T = 64, 32, 3
    arr = _rand_layer(rng, H, I, 1, 0, bits=bits)
    x_bits = synth.normal_bf16(9, 0, 1, (T, H))
    r = cr.moe_layer(arr, x_bits, 1, 1, 0, bits=bits, logits_in=np.zeros((T, 1), np.float32))
    Wg, Wu, Wd = (_py_dequant(*(a[0] for a in arr[kk]), bits=bits) for kk in ("gate", "up", "down"))
    for t in range(T):
        ref = _py_dense_swiglu(oracle.bf16_bits_to_f64(x_bits[t]).tolist(), Wg, Wu, Wd)
        assert np.allclose(r["acc"][t], ref, rtol=1e-12, atol=1e-12 * max(map(abs, ref)))


def test_shared_expert_alone_is_dense():
    """Routed experts with zero codes: the output is the shared expert's dense FFN."""
    rng = np.random.default_rng(28)
    H, I, E, T = 64, 32, 4, 2
    arr = _rand_layer(rng, H, I, E, 1, zero_routed=True)
    x_bits = synth.normal_bf16(10, 0, 1, (T, H))
    r = cr.moe_layer(arr, x_bits, E, 2, 1, logits_in=rng.standard_normal((T, E)).astype(np.float32))
    Wg, Wu, Wd = (_py_dequant(*(a[E] for a in arr[kk])) for kk in ("gate", "up", "down"))
    for t in range(T):
        ref = _py_dense_swiglu(oracle.bf16_bits_to_f64(x_bits[t]).tolist(), Wg, Wu, Wd)
        assert np.allclose(r["acc"][t], ref, rtol=1e-12, atol=1e-12 * max(map(abs, ref)))


def test_combine_is_routing_weighted_sum_of_dense_experts():
    """E=3, k=2: out = w0 * dense_{id0}(x) + w1 * dense_{id1}(x) + residual."""
    rng = np.random.default_rng(29)
    H, I, E, T = 32, 32, 3, 3
    arr = _rand_layer(rng, H, I, E, 0)
    x_bits = synth.normal_bf16(11, 0, 1, (T, H))
    res_bits = synth.normal_bf16(12, 0, 1, (T, H))
    r = cr.moe_layer(arr, x_bits, E, 2, 0, logits_in=rng.standard_normal((T, E)).astype(np.float32),
                     residual_bits=res_bits)
    dense = [[_py_dequant(*(a[e] for a in arr[kk])) for kk in ("gate", "up", "down")] for e in range(E)]
    for t in range(T):
        x = oracle.bf16_bits_to_f64(x_bits[t]).tolist()
        ref = np.array(oracle.bf16_bits_to_f64(res_bits[t]))
        for j in range(2):
            ref = ref + r["w"][t, j] * np.array(_py_dense_swiglu(x, *dense[r["ids"][t, j]]))
        assert np.allclose(r["acc"][t], ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_zero_codes_give_residual_and_down_scale_doubles_output():
    rng = np.random.default_rng(30)
    H, I, E, S, T = 64, 32, 4, 1, 3
    arr = _rand_layer(rng, H, I, E, S)
    x_bits = synth.normal_bf16(13, 0, 1, (T, H))
    res = synth.normal_bf16(14, 0, 1, (T, H))
    lg = rng.standard_normal((T, E)).astype(np.float32)
    zero = {kk: (np.zeros_like(v[0]), v[1]) for kk, v in arr.items()}
    assert np.array_equal(cr.moe_layer(zero, x_bits, E, 2, S, logits_in=lg, residual_bits=res)["out"], res)
    a1 = cr.moe_layer(arr, x_bits, E, 2, S, logits_in=lg)["acc"]
    s2 = (arr["down"][1].view(np.float16).astype(np.float32) * 2).astype(np.float16).view(np.uint16)
    a2 = cr.moe_layer(dict(arr, down=(arr["down"][0], s2)), x_bits, E, 2, S, logits_in=lg)["acc"]
    assert np.array_equal(a2, 2 * a1)


def test_ffn_one_code_hand_worked():
    g = {ln.split()[0]: ln for ln in _golden("ffn_one_code.txt")}
    H = I = 32
    arr = {kk: (np.zeros((1, r, K // 2), np.uint8), np.zeros((1, r, K // 32), np.uint16))
           for kk, (r, K) in {"gate": (I, H), "up": (I, H), "down": (H, I)}.items()}
    for kind in ("gate", "up", "down"):
        _, r, c, code, sbits = g[kind].split()
        r, c, code = int(r), int(c), int(code)
        arr[kind][0][0, r, c // 2] |= (code & 0xF) << (4 * (c % 2))
        arr[kind][1][0, r, c // 32] = int(sbits, 16)
    x = np.zeros((1, H), np.float32)
    x[0, 3] = 2.0
    out = cr.moe_layer(arr, synth.f32_to_bf16_bits(x), 1, 1, 0, logits_in=np.zeros((1, 1), np.float32))["out"]
    want = np.zeros(H)
    _, r, v = g["out"].split()
    want[int(r)] = float(v)
    assert oracle.bf16_bits_to_f64(out[0]).tolist() == want.tolist()


def test_rms_norm_matches_library():
    h = synth.normal_bf16(16, 0, 1, (5, 256))
    ref = torch.nn.functional.rms_norm(torch.from_numpy(oracle.bf16_bits_to_f64(h)), (256,), eps=oracle.RMS_EPS)
    assert np.array_equal(cr.decode_bf16(cr.rms_norm(h)), cr.round_bf16(ref.numpy()))


def _arrays(rng, H, I, n, group, bits):
    arr = {}
    for kind, (r, K) in {"gate": (I, H), "up": (I, H), "down": (H, I)}.items():
        c = rng.integers(0, 256, size=(n, r, K * bits // 8), dtype=np.uint8)
        s = rng.uniform(0.004, 0.02, size=(n, r, K // group)).astype(np.float16).view(np.uint16)
        arr[kind] = (c, s)
    return arr


def _assert_outputs_agree(out_c, acc_c, out_n, acc_n):
    """Sums within 1e-12 of max|sum|; bf16 outputs equal, except an element whose
    sum sits within that distance of the midpoint between the two values."""
    tol = 1e-12 * np.abs(acc_n).max(initial=1e-300)
    assert np.abs(acc_c - acc_n).max(initial=0.0) <= tol
    d = np.nonzero(out_c != out_n)
    if d[0].size:
        a, b = oracle.bf16_bits_to_f64(out_c[d]), oracle.bf16_bits_to_f64(out_n[d])
        assert np.all(np.abs(acc_n[d] - (a + b) / 2) <= tol)


CASES = [  # T, H, I, E, k, S, group, bits, bias, residual
    (1, 64, 32, 8, 2, 1, 32, 4, False, False),
    (5, 128, 64, 6, 3, 0, 64, 4, True, False),
    (7, 64, 64, 16, 4, 2, 32, 8, False, True),
    (37, 128, 64, 12, 8, 1, 64, 8, True, True),
    (20, 256, 128, 32, 8, 1, 32, 4, True, True),
    (0, 64, 32, 8, 2, 1, 32, 4, False, False),
]


@pytest.mark.parametrize("T,H,I,E,k,S,group,bits,use_bias,use_res", CASES)
def test_c_oracle_agrees_with_numpy_oracle(T, H, I, E, k, S, group, bits, use_bias, use_res):
    rng = np.random.default_rng(1000 + T * 31 + H + E)
    arr = _arrays(rng, H, I, E + S, group, bits)
    x = synth.normal_bf16(30 + T, 1, 1, (T, H))
    rw = (rng.standard_normal((E, H)) * 0.05).astype(np.float32)
    bias = (rng.standard_normal(E) * 0.5).astype(np.float32) if use_bias else None
    res = synth.normal_bf16(40 + T, 2, 1, (T, H)) if use_res else None
    rc = cr.moe_layer(arr, x, E, k, S, group, bits, router_w=rw, bias=bias, residual_bits=res)
    W = oracle.ExpertWeights.from_arrays(arr, group, bits)
    rn = oracle.moe_layer(W, x, E, k, S, router_w=rw, bias=bias, residual_bits=res)
    assert np.allclose(rc["logits64"], rn["logits64"], rtol=0, atol=1e-13 * np.abs(rn["logits64"]).max(initial=1.0))
    assert np.array_equal(rc["logits32"], rn["logits32"])
    assert np.array_equal(rc["ids"], rn["ids"])
    assert np.allclose(rc["w"], rn["w"], rtol=1e-14, atol=0)
    assert np.array_equal(rc["flags"], rn["flags"])
    _, acc_n = oracle.moe_ffn_combine(W, x, rn["ids"], rn["w"], E, S, residual_bits=res, return_f64=True)
    _assert_outputs_agree(rc["out"], rc["acc"], rn["out"], acc_n)


def test_c_oracle_agrees_on_given_logits_with_ties():
    """Routing from given fp32 logits full of ties: ids and weights identical."""
    rng = np.random.default_rng(50)
    T, H, I, E, k, S = 24, 64, 32, 10, 4, 1
    arr = _arrays(rng, H, I, E + S, 32, 4)
    x = synth.normal_bf16(51, 0, 1, (T, H))
    lg = rng.integers(-2, 3, size=(T, E)).astype(np.float32)
    rc = cr.moe_layer(arr, x, E, k, S, logits_in=lg)
    W = oracle.ExpertWeights.from_arrays(arr)
    rn = oracle.moe_layer(W, x, E, k, S, logits_in=lg)
    assert np.array_equal(rc["ids"], rn["ids"])
    assert np.array_equal(rc["w"], rn["w"]) or np.allclose(rc["w"], rn["w"], rtol=1e-15, atol=0)
    _, acc_n = oracle.moe_ffn_combine(W, x, rn["ids"], rn["w"], E, S, return_f64=True)
    _assert_outputs_agree(rc["out"], rc["acc"], rn["out"], acc_n)


def test_c_oracle_stack_agrees_with_numpy_oracle():
    """Two stacked layers, h_{l+1} = bf16(h_l + MoE_l(rms_norm(h_l)))."""
    rng = np.random.default_rng(60)
    H, I, E, k, S, T = 64, 32, 8, 2, 1, 4
    layers = [(_arrays(rng, H, I, E + S, 32, 4), (rng.standard_normal((E, H)) * 0.1).astype(np.float32))
              for _ in range(2)]
    h0 = synth.normal_bf16(61, 0, 1, (T, H))
    hn, _ = oracle.moe_stack([(oracle.ExpertWeights.from_arrays(a), rw, None) for a, rw in layers], h0, E, k, S)
    h = h0
    for a, rw in layers:
        h = cr.moe_layer(a, cr.rms_norm(h), E, k, S, router_w=rw, residual_bits=h)["out"]
    assert np.array_equal(h, hn)


def test_layer_rejects_bad_arguments():
    rng = np.random.default_rng(70)
    arr = _arrays(rng, 64, 32, 3, 32, 4)
    x = synth.normal_bf16(71, 0, 1, (2, 64))
    with pytest.raises(ValueError):
        cr.moe_layer(arr, x, 2, 3, 1, logits_in=np.zeros((2, 2), np.float32))     # k > E
    with pytest.raises(ValueError):
        cr.moe_layer(arr, x, 2, 1, 1)                                               # no logits, no router


def _brute_topk_fast(l, k):
    """All k-subsets S of range(E); keep those whose weakest member beats the
    strongest non-member under (value descending, index ascending)."""
    E = len(l)
    rank = lambda e: (-l[e], e)  # noqa: E731  smaller is stronger
    found = []
    for S in itertools.combinations(range(E), k):
        inside = set(S)
        weakest = max(S, key=rank)
        if all(rank(weakest) < rank(j) for j in range(E) if j not in inside):
            found.append(set(S))
    assert len(found) == 1
    return found[0]


def test_route_matches_brute_force_up_to_16_experts_both_oracles():
    rng = np.random.default_rng(31)
    for _ in range(40):
        E = int(rng.integers(9, 17))
        k = int(rng.integers(1, 9))
        l = rng.integers(0, 4, size=(1, E)).astype(np.float32)
        want = _brute_topk_fast(l[0].tolist(), k)
        for ids in (cr.route(l, k)[0], oracle.route(l, k)[0]):
            assert set(ids[0].tolist()) == want
            assert [(-l[0, e], e) for e in ids[0]] == sorted((-l[0, e], e) for e in ids[0])


@pytest.mark.slow
def test_c_oracle_agrees_with_numpy_oracle_at_glm_size():
    """One token of the GLM-shaped layer (H 6144, I 2048, 256 experts, k 8, one
    shared expert) with the Zipf bias and a residual: the C oracle fetches only
    the experts the token selects."""
    shape = synth.DECODE_B64
    li = synth.LayerInputs(shape)
    kinds = {"gate": (synth.GATE_Q, synth.GATE_S), "up": (synth.UP_Q, synth.UP_S), "down": (synth.DOWN_Q, synth.DOWN_S)}
    x = synth.activations(shape)[:1]
    rw, bias = li.router_w(), li.bias()
    assert bias is not None
    rc = cr.moe_layer_experts(lambda kind, e: (li.expert_codes(kinds[kind][0], e), li.expert_scales(kinds[kind][1], e)),
                              shape.hidden, shape.inter, x, shape.n_experts, shape.top_k, shape.n_shared, shape.group,
                              shape.bits, router_w=rw, bias=bias, residual_bits=x)
    W = oracle.ExpertWeights.from_synth(li)
    rn = oracle.moe_layer(W, x, shape.n_experts, shape.top_k, shape.n_shared, router_w=rw, bias=bias, residual_bits=x)
    assert np.array_equal(rc["logits32"], rn["logits32"]) and np.array_equal(rc["ids"], rn["ids"])
    assert np.allclose(rc["w"], rn["w"], rtol=1e-14, atol=0)
    _, acc_n = oracle.moe_ffn_combine(W, x, rn["ids"], rn["w"], shape.n_experts, shape.n_shared, residual_bits=x,
                                      return_f64=True)
    _assert_outputs_agree(rc["out"], rc["acc"], rn["out"], acc_n)


def test_lazy_layer_matches_and_rejects_a_missing_selected_expert():
    """The per-expert entry gives the contiguous entry's bits, and refuses to
    run when an expert the batch selected was not given."""
    rng = np.random.default_rng(80)
    arr = _arrays(rng, 64, 32, 5, 32, 4)
    x = synth.normal_bf16(81, 0, 1, (3, 64))
    lg = rng.standard_normal((3, 4)).astype(np.float32)
    fetch = lambda kind, e: (arr[kind][0][e], arr[kind][1][e])  # noqa: E731
    r = cr.moe_layer_experts(fetch, 64, 32, x, 4, 2, 1, logits_in=lg)
    full = cr.moe_layer(arr, x, 4, 2, 1, logits_in=lg)
    assert np.array_equal(r["out"], full["out"]) and np.array_equal(r["acc"], full["acc"])
    picked = set(r["ids"].ravel().tolist())
    for missing in sorted(picked) + [4]:                 # a routed expert, then the shared one
        with pytest.raises(ValueError):
            cr.moe_layer_experts(fetch, 64, 32, x, 4, 2, 1, logits_in=lg, experts=(picked | {4}) - {missing})


def test_oracles_agree_on_random_small_layers():
    """Property check over random shapes, containers, biases, residuals and
    logit styles (computed, given with dense ties, given with NaN/inf)."""
    from hypothesis import given, settings, HealthCheck
    from hypothesis import strategies as st

    @settings(max_examples=100, deadline=None, derandomize=True, suppress_health_check=list(HealthCheck))
    @given(T=st.integers(0, 6), E=st.integers(1, 12), kfrac=st.floats(0, 1), S=st.integers(0, 2),
           group=st.sampled_from([32, 64]), bits=st.sampled_from([4, 8]), hmul=st.integers(1, 2),
           imul=st.integers(1, 2), logits=st.sampled_from(["router", "ties", "nonfinite"]),
           use_bias=st.booleans(), use_res=st.booleans(), seed=st.integers(0, 2 ** 31 - 1))
    def check(T, E, kfrac, S, group, bits, hmul, imul, logits, use_bias, use_res, seed):
        rng = np.random.default_rng(seed)
        k = 1 + int(kfrac * (E - 1))
        H, I = 64 * hmul, 64 * imul
        arr = _arrays(rng, H, I, E + S, group, bits)
        x = synth.normal_bf16(seed % 1000, 3, 1, (T, H))
        rw = lg = None
        if logits == "router":
            rw = (rng.standard_normal((E, H)) * 0.1).astype(np.float32)
        else:
            lg = rng.integers(-2, 3, size=(T, E)).astype(np.float32)
            if logits == "nonfinite" and T:
                lg[0, rng.integers(E)] = [np.nan, np.inf, -np.inf][int(rng.integers(3))]
        bias = (rng.standard_normal(E) * 0.5).astype(np.float32) if use_bias else None
        res = synth.normal_bf16(seed % 1000, 4, 1, (T, H)) if use_res else None
        rc = cr.moe_layer(arr, x, E, k, S, group, bits, router_w=rw, logits_in=lg, bias=bias, residual_bits=res)
        W = oracle.ExpertWeights.from_arrays(arr, group, bits)
        rn = oracle.moe_layer(W, x, E, k, S, router_w=rw, logits_in=lg, bias=bias, residual_bits=res)
        assert np.array_equal(rc["ids"], rn["ids"]) and np.array_equal(rc["flags"], rn["flags"])
        assert np.array_equal(rc["logits32"], rn["logits32"], equal_nan=True)
        if rn["flags"].any():
            return                      # weights and outputs are not meaningful for flagged tokens
        assert np.allclose(rc["w"], rn["w"], rtol=1e-14, atol=0)
        _, acc_n = oracle.moe_ffn_combine(W, x, rn["ids"], rn["w"], E, S, residual_bits=res, return_f64=True)
        _assert_outputs_agree(rc["out"], rc["acc"], rn["out"], acc_n)

    check()
