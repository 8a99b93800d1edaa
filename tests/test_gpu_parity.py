"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Routing ids, union lists and permutations: bit-exact when both sides route
from the same fp32 logits.  Floating-point outputs: within the tolerances of
``tests/_gpu.py``.  The decode batch-1 layer is compared in full here; the
other full-size workloads (many tokens, every stack layer) are in
``tests/test_gpu_fullsize.py``.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._gpu import (OUT_REL_TOL, ambiguous_tokens, bits, device_layer, logits_tol, needs_gpu, oracle_weights,
                        route_w_tol, to_dev_bits)

pytestmark = [pytest.mark.gpu, needs_gpu]


@pytest.fixture(scope="module")
def lib():
    import int4_routed_expert_renorm_b200 as m
    m.coli_moe_get_status()  # clear any stale bits
    return m


def _status(lib):
    st, flags = lib.coli_moe_get_status()
    return flags


# ---------------------------------------------------------------- generator

@pytest.mark.parametrize("shape", [synth.TINY, synth.DECODE_B1], ids=lambda s: s.name)
def test_device_fill_matches_numpy_generator(shape):
    import synth.gpu as sg
    t = sg.expert_tensors(shape)
    li = synth.LayerInputs(shape)
    for e in sorted({0, 1, shape.n_total - 1, shape.n_total // 2}):
        for name, qk, sk in (("gate", synth.GATE_Q, synth.GATE_S), ("up", synth.UP_Q, synth.UP_S),
                             ("down", synth.DOWN_Q, synth.DOWN_S)):
            assert np.array_equal(t[name + "_q"][e].cpu().numpy(), li.expert_codes(qk, e))
            assert np.array_equal(t[name + "_s"][e].cpu().numpy().view(np.uint16), li.expert_scales(sk, e))
    del t
    torch.cuda.empty_cache()


# ---------------------------------------------------------------- route

def _route_case(lib, l32, k, bias=None):
    T, E = l32.shape
    lg = torch.from_numpy(l32).cuda()
    b = None if bias is None else torch.from_numpy(bias).cuda()
    ids = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    w = torch.full((T, k), -7.0, dtype=torch.float32, device="cuda")
    lib.coli_moe_route(lg, b, ids, w)
    flags = _status(lib)
    rid, rw, rflags = oracle.route(oracle.add_bias(l32, bias), k)
    return ids.cpu().numpy(), w.cpu().numpy(), flags, rid, rw, rflags


@pytest.mark.parametrize("T,E,k,kind", [
    (4, 16, 2, "normal"), (1, 256, 8, "normal"), (64, 256, 8, "zipf"), (4096, 256, 8, "normal"),
    (37, 1024, 32, "normal"), (500, 64, 8, "ties"), (300, 16, 1, "ties"), (9, 16, 16, "normal"),
    (33, 33, 5, "ties"), (0, 16, 2, "normal")])
def test_route_bit_exact(lib, T, E, k, kind):
    rng = np.random.default_rng(T * 7919 + E * 31 + k)
    if kind == "ties":
        l32 = rng.integers(0, 4, size=(T, E)).astype(np.float32)
        l32[rng.random((T, E)) < 0.1] = -0.0
    else:
        l32 = rng.standard_normal((T, E)).astype(np.float32)
    bias = synth.zipf_bias(0, 0, E) if kind == "zipf" else None
    ids, w, flags, rid, rw, rflags = _route_case(lib, l32, k, bias)
    assert flags == 0
    assert np.array_equal(ids, rid)
    assert np.abs(w - rw).max(initial=0) <= route_w_tol(k)


def test_route_nonfinite_sets_flag(lib):
    l32 = np.random.default_rng(1).standard_normal((6, 32)).astype(np.float32)
    l32[1, 5] = np.nan
    l32[3, 0] = np.inf
    l32[4, :] = -np.inf
    l32[4, 7] = 1.0
    ids, w, flags, rid, rw, rflags = _route_case(lib, l32, 4)
    assert flags & lib._lib.COLI_FLAG_NONFINITE
    assert np.array_equal(ids, rid)                 # selection still defined (NaN ranks as -inf)
    clean = rflags == 0
    assert np.abs(w[clean] - rw[clean]).max() <= route_w_tol(4)


# ---------------------------------------------------------------- union

def _union_case(lib, ids_np, E):
    T, k = ids_np.shape
    P = T * k
    Umax = max(1, min(E, P))
    d = torch.from_numpy(ids_np.astype(np.int32)).cuda()
    uq = torch.full((Umax,), -5, dtype=torch.int32, device="cuda")
    nu = torch.full((1,), -5, dtype=torch.int32, device="cuda")
    so = torch.full((Umax + 1,), -5, dtype=torch.int32, device="cuda")
    pm = torch.full((max(P, 1),), -5, dtype=torch.int32, device="cuda")
    pp = torch.full((max(P, 1),), -5, dtype=torch.int32, device="cuda")
    lib.coli_moe_union(d, E, uq, nu, so, pm, pp)
    flags = _status(lib)
    U = int(nu.item())
    return (uq.cpu().numpy()[:U], U, so.cpu().numpy()[:U + 1], pm.cpu().numpy()[:P], pp.cpu().numpy()[:P], flags)


@pytest.mark.parametrize("T,E,k,dist", [(1, 256, 8, "u"), (4, 16, 2, "u"), (64, 256, 8, "zipf"),
                                        (4096, 256, 8, "u"), (300, 16, 2, "hot"), (7, 1024, 32, "u"),
                                        (2048, 1024, 8, "u"), (0, 16, 2, "u")])
def test_union_bit_exact(lib, T, E, k, dist):
    rng = np.random.default_rng(T + E + k)
    if dist == "hot":  # expert 3 in every token
        ids = np.array([[3] + list(rng.choice([e for e in range(E) if e != 3], k - 1, replace=False))
                        for _ in range(T)]).reshape(T, k)
    elif dist == "zipf":
        p = np.arange(1, E + 1, dtype=np.float64) ** -1.1
        ids = np.array([rng.choice(E, k, replace=False, p=p / p.sum()) for _ in range(T)]).reshape(T, k)
    else:
        ids = np.array([rng.choice(E, k, replace=False) for _ in range(T)]).reshape(T, k)
    uq, U, so, pm, pp, flags = _union_case(lib, ids, E)
    ru, rs, rp, rpp = oracle.batch_union(ids, E)
    assert flags == 0
    assert U == len(ru)
    assert np.array_equal(uq, ru) and np.array_equal(so, rs)
    assert np.array_equal(pm, rp) and np.array_equal(pp, rpp)


def test_union_bad_id_flag(lib):
    ids = np.array([[1, 2], [3, 99], [1, -1]], np.int32)
    uq, U, so, pm, pp, flags = _union_case(lib, ids, 16)
    assert flags & lib._lib.COLI_FLAG_BAD_ID
    assert pp[3] == -1 and pp[5] == -1
    assert uq.tolist() == [1, 2, 3] and so.tolist() == [0, 2, 3, 4]


# ---------------------------------------------------------------- whole layer

def run_gpu_layer(lib, layer, x_bits, logits_in=None, residual_bits=None, flags=0):
    T = x_bits.shape[0]
    d = layer.dims
    x = to_dev_bits(x_bits)
    out = torch.empty_like(x)
    ws = layer.workspace(T)
    lo = torch.empty((T, d.n_experts), dtype=torch.float32, device="cuda")
    ids = torch.empty((T, d.top_k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, d.top_k), dtype=torch.float32, device="cuda")
    li = None if logits_in is None else torch.from_numpy(logits_in).cuda()
    res = None if residual_bits is None else to_dev_bits(residual_bits)
    layer.forward(x, out, ws, logits_in=li, residual=res, flags=flags, logits_out=lo, topk_ids_out=ids,
                  topk_w_out=w)
    st = _status(lib)
    return dict(out=bits(out), logits=lo.cpu().numpy(), ids=ids.cpu().numpy(), w=w.cpu().numpy(), flags=st)


def check_layer(lib, shape, layer, W, x_bits, sample=None, logits_in=None, residual_bits=None, rw=None,
                bias=None, flags=0, max_ambiguous=0):
    """Run the GPU layer and compare with the oracle; returns the observed relative error."""
    g = run_gpu_layer(lib, layer, x_bits, logits_in, residual_bits, flags)
    assert g["flags"] == 0, g["flags"]
    T, k = x_bits.shape[0], shape.top_k
    xin = oracle.rms_norm(x_bits) if flags & lib._lib.COLI_LAYER_PRENORM else x_bits
    if logits_in is None:
        l64, l32 = oracle.router_logits(xin, rw)
        tol = logits_tol(xin, rw)
        assert np.all(np.abs(g["logits"] - l64) <= tol), np.abs(g["logits"] - l64).max()
        amb = ambiguous_tokens(l32, tol, bias, k)
    else:
        l32 = logits_in
        assert np.array_equal(g["logits"], logits_in)
        amb = np.zeros(T, bool)
    assert amb.sum() <= max_ambiguous
    rid, rwt, rfl = oracle.route(oracle.add_bias(l32, bias), k)
    ok = ~amb
    assert np.array_equal(g["ids"][ok], rid[ok])
    assert np.abs(g["w"][ok] - rwt[ok]).max(initial=0) <= route_w_tol(k) + 1e-5
    toks = np.arange(T) if sample is None else np.asarray(sample)
    toks = toks[ok[toks]]
    res = None if residual_bits is None else residual_bits[toks]
    ref = oracle.moe_ffn_combine(W, xin[toks], rid[toks], rwt[toks], shape.n_experts, shape.n_shared, res)
    got = oracle.bf16_bits_to_f64(g["out"][toks])
    want = oracle.bf16_bits_to_f64(ref)
    err = np.abs(got - want).max() / np.abs(want).max()
    assert np.isfinite(got).all()
    assert err <= OUT_REL_TOL, err
    return err, g


def _small_shape(**kw):
    d = dict(name="small", hidden=256, inter=128, n_experts=16, top_k=2, n_shared=0, tokens=4)
    d.update(kw)
    return synth.LayerShape(**d)


def test_layer_tiny_workload(lib):
    shape = synth.TINY
    layer = device_layer(shape)
    li = synth.LayerInputs(shape)
    err, g = check_layer(lib, shape, layer, oracle_weights(shape), synth.activations(shape), rw=li.router_w())
    assert err < 1e-2


@pytest.mark.parametrize("kw", [
    dict(tokens=1), dict(tokens=5), dict(tokens=13, n_shared=1), dict(tokens=67, n_shared=1),
    dict(tokens=9, top_k=1), dict(tokens=6, top_k=16), dict(tokens=20, inter=256, n_shared=2),
    dict(tokens=3, hidden=512, inter=256, n_experts=40, top_k=5, n_shared=1)],
    ids=lambda kw: "-".join(f"{k}{v}" for k, v in kw.items()))
def test_layer_ragged_shapes(lib, kw):
    shape = _small_shape(**kw)
    layer = device_layer(shape, seed=3)
    li = synth.LayerInputs(shape, seed=3)
    x = synth.normal_bf16(3, 5, synth.X_IN, (shape.tokens, shape.hidden))
    res = synth.normal_bf16(3, 6, synth.X_IN, (shape.tokens, shape.hidden))
    check_layer(lib, shape, layer, oracle_weights(shape, seed=3), x, rw=li.router_w(), residual_bits=res)


def test_layer_hot_expert_300_tokens(lib):
    """One expert receives all 300 tokens (several 64-token blocks), logits given."""
    shape = _small_shape(tokens=300, n_shared=1)
    layer = device_layer(shape, seed=4)
    rng = np.random.default_rng(4)
    l = rng.standard_normal((300, 16)).astype(np.float32)
    l[:, 3] += 50.0
    x = synth.normal_bf16(4, 5, synth.X_IN, (300, shape.hidden))
    check_layer(lib, shape, layer, oracle_weights(shape, seed=4), x, logits_in=l)


def test_layer_prenorm_and_expert_ffn_call(lib):
    """Pre-norm layer; and route + union + expert_ffn called separately give the
    same bits as the layer call."""
    shape = _small_shape(tokens=11, n_shared=1)
    layer = device_layer(shape, seed=5)
    li = synth.LayerInputs(shape, seed=5)
    x = synth.normal_bf16(5, 5, synth.X_IN, (11, shape.hidden))
    err, g = check_layer(lib, shape, layer, oracle_weights(shape, seed=5), x, rw=li.router_w(), residual_bits=x,
                         flags=lib._lib.COLI_LAYER_PRENORM)
    # separate calls on the same routed batch (no pre-norm)
    g2 = run_gpu_layer(lib, layer, x)
    d = layer.dims
    xd = to_dev_bits(x)
    ids = torch.from_numpy(g2["ids"]).cuda()
    w = torch.from_numpy(g2["w"]).cuda()
    P = 11 * d.top_k
    U = min(d.n_experts, P)
    uq = torch.empty(U, dtype=torch.int32, device="cuda")
    nu = torch.empty(1, dtype=torch.int32, device="cuda")
    so = torch.empty(U + 1, dtype=torch.int32, device="cuda")
    pm = torch.empty(P, dtype=torch.int32, device="cuda")
    pp = torch.empty(P, dtype=torch.int32, device="cuda")
    lib.coli_moe_union(ids, d.n_experts, uq, nu, so, pm, pp)
    out = torch.empty_like(xd)
    ws = layer.workspace(11)
    lib.coli_moe_expert_ffn(d, layer.weights, xd, ids, w, uq, nu, so, pm, pp, None, out, ws)
    assert _status(lib) == 0
    assert np.array_equal(bits(out), g2["out"])


# ---------------------------------------------------------------- full-size workloads

@pytest.fixture(scope="module")
def glm_layer():
    layer = device_layer(synth.DECODE_B1)
    yield layer
    del layer
    torch.cuda.empty_cache()


def test_glm_decode_b1_full(lib, glm_layer):
    shape = synth.DECODE_B1
    li = synth.LayerInputs(shape)
    err, g = check_layer(lib, shape, glm_layer, oracle_weights(shape), synth.activations(shape),
                         rw=li.router_w())
    print(f"decode b1: max rel err {err:.3e}")


# ---------------------------------------------------------------- batch invariance

@pytest.mark.parametrize("prenorm", [False, True], ids=["plain", "prenorm"])
def test_router_logits_do_not_depend_on_the_batch_glm(lib, glm_layer, prenorm):
    """Batches of up to 8 tokens get their router logits from front_kernel,
    larger ones from logits_tile_kernel.  Both sum every (token, expert) dot
    product in the same order, so a token's logits, and with them its
    routing, are the same bits in a batch of 12 as alone."""
    shape = synth.DECODE_B1
    x = np.concatenate([synth.activations(shape, 0, b) for b in range(12)])
    flags = lib._lib.COLI_LAYER_PRENORM if prenorm else 0
    gb = run_gpu_layer(lib, glm_layer, x, flags=flags)
    assert gb["flags"] == 0
    for t in (0, 5, 11):
        g1 = run_gpu_layer(lib, glm_layer, x[t:t + 1], flags=flags)
        assert np.array_equal(g1["logits"][0], gb["logits"][t]), t
        assert np.array_equal(g1["ids"][0], gb["ids"][t]) and np.array_equal(g1["w"][0], gb["w"][t]), t


@pytest.mark.parametrize("hidden", [256, 512, 768, 1280])
def test_router_logits_do_not_depend_on_the_batch_small(lib, hidden):
    """The same across H whose eighth is not a multiple of 128 (some lanes of
    each range idle, ragged last chunk)."""
    shape = _small_shape(tokens=20, hidden=hidden, inter=128, n_experts=24, top_k=3)
    layer = device_layer(shape, seed=14)
    x = synth.normal_bf16(14, 5, synth.X_IN, (20, hidden))
    gb = run_gpu_layer(lib, layer, x)
    for t in range(0, 20, 3):
        g1 = run_gpu_layer(lib, layer, x[t:t + 1])
        assert np.array_equal(g1["logits"][0], gb["logits"][t]), t
    g8 = run_gpu_layer(lib, layer, x[:8])
    assert np.array_equal(g8["logits"], gb["logits"][:8])


@pytest.mark.parametrize("kw", [dict(tokens=70, hidden=512, n_experts=24, top_k=3),
                                dict(tokens=130, hidden=768, n_experts=100, top_k=8, n_shared=1)],
                         ids=lambda kw: "-".join(f"{k}{v}" for k, v in kw.items()))
def test_router_logits_tensor_core_path(lib, kw):
    """Batches of 65 tokens or more get their router logits from the tensor
    cores (three bf16 pieces of W_r): every logit within the fp32 bound of the
    float64 oracle, routing and output checked as everywhere (tile edges: T
    and E not multiples of 64); and a token's logits are the same bits in a
    batch of 65 as in the larger one."""
    shape = _small_shape(**kw)
    layer = device_layer(shape, seed=15)
    li = synth.LayerInputs(shape, seed=15)
    x = synth.normal_bf16(15, 5, synth.X_IN, (shape.tokens, shape.hidden))
    err, g = check_layer(lib, shape, layer, oracle_weights(shape, seed=15), x, rw=li.router_w(), max_ambiguous=2)
    l64, _ = oracle.router_logits(x, li.router_w())
    xa = np.abs(synth.bf16_bits_to_f32(x).astype(np.float64)) @ np.abs(li.router_w().astype(np.float64)).T
    print(f"tensor-core logits: max error {np.abs(g['logits'] - l64).max():.2e}, "
          f"in units of 2^-24 sum|x w|: {(np.abs(g['logits'] - l64) / (2.0 ** -24 * xa)).max():.2f}")
    g65 = run_gpu_layer(lib, layer, x[:65])
    assert np.array_equal(g65["logits"], g["logits"][:65])


@pytest.mark.parametrize("T", [2, 4, 8])
def test_decode_batch_invariance(lib, glm_layer, T):
    """A token's output in a batch of T (draft + verify tokens decoded in one
    forward) is bit-identical to its output when decoded alone: each token's
    dot products, group scaling, K-half reduction and combine run in the same
    order whatever the batch, and routing is per token."""
    shape = synth.DECODE_B1
    x = np.concatenate([synth.activations(shape, 0, b) for b in range(T)])
    gb = run_gpu_layer(lib, glm_layer, x, residual_bits=x, flags=lib._lib.COLI_LAYER_PRENORM)
    assert gb["flags"] == 0
    for t in range(T):
        g1 = run_gpu_layer(lib, glm_layer, x[t:t + 1], residual_bits=x[t:t + 1], flags=lib._lib.COLI_LAYER_PRENORM)
        assert np.array_equal(g1["ids"][0], gb["ids"][t])
        assert np.array_equal(g1["out"][0], gb["out"][t]), t


@pytest.mark.parametrize("inter", [256, 512])
def test_two_phase_form_is_batch_invariant(lib, inter):
    """Batches of 9..64 tokens run 16-token tiles, larger ones 32-token tiles:
    the tokens a 65-token batch shares with a 64-token and a 9-token batch get
    the same bits (per-token MMA columns and fixed reduction orders), with one
    and with two 256-wide down K chunks."""
    shape = _small_shape(tokens=65, hidden=512, inter=inter, n_experts=8, top_k=2, n_shared=1)
    layer = device_layer(shape, seed=13)
    x = synth.normal_bf16(13, 5, synth.X_IN, (65, shape.hidden))
    # logits given, so that routing does not depend on which logits kernel the batch size picks
    lg = np.random.default_rng(13).standard_normal((65, shape.n_experts)).astype(np.float32)
    g65 = run_gpu_layer(lib, layer, x, logits_in=lg, residual_bits=x)
    g64 = run_gpu_layer(lib, layer, x[:64], logits_in=lg[:64], residual_bits=x[:64])
    g9 = run_gpu_layer(lib, layer, x[:9], logits_in=lg[:9], residual_bits=x[:9])
    assert g65["flags"] == g64["flags"] == g9["flags"] == 0
    assert np.array_equal(g65["ids"][:64], g64["ids"])
    assert np.array_equal(g65["out"][:64], g64["out"])
    assert np.array_equal(g65["out"][:9], g9["out"])
