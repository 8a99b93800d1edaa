"""Full-size parity with the plain-C oracle on many tokens.

The GLM-5.2-shaped workloads (H 6144, I 2048, 256 experts, top-8, one shared
expert) through the C ABI, against the C oracle run token by token over the
host's cores (tests/_cref_pool.py), each call reading only the experts its
token selects.  Both sides route from the same fp32 logits -- the GPU's own,
which are checked against the oracle's logits within the derived fp32 bound,
or the workload's given logits -- so routing ids are compared bit-exactly
and every output element within 1e-2 of the largest reference magnitude
(the layer statement's bar):
  * decode, batch 64 with the Zipf router bias: all 64 tokens;
  * prefill, 4096 tokens: at least 64 tokens, among them the first and the
    last token of every token block (the prefill form cuts a segment into
    blocks of at most 160 tokens) of the two hottest and the two coldest
    experts, and the first and last token of the batch; the prefill form
    and the decode form (forced) on the same tokens;
  * the 16-layer stack at batch 4 with pre-norm and residual: every layer,
    teacher-forced on the hidden state the GPU produced for it.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._cref_pool import layer_jobs, layer_outputs
from tests._gpu import OUT_REL_TOL, bits, device_layer, logits_tol, needs_gpu, to_dev_bits

pytestmark = [pytest.mark.gpu, needs_gpu]

PRENORM, DECODE, PREFILL = 0x1, 0x10, 0x20


@pytest.fixture(scope="module")
def lib():
    import int4_routed_expert_renorm_b200 as m
    m.coli_moe_get_status()
    return m


def _gpu_layer(lib, layer, x_bits, logits_in=None, residual_bits=None, flags=0):
    T, d = x_bits.shape[0], layer.dims
    x = to_dev_bits(x_bits)
    out = torch.empty_like(x)
    lo = torch.empty((T, d.n_experts), dtype=torch.float32, device="cuda")
    ids = torch.empty((T, d.top_k), dtype=torch.int32, device="cuda")
    li = None if logits_in is None else torch.from_numpy(logits_in).cuda()
    res = None if residual_bits is None else to_dev_bits(residual_bits)
    layer.forward(x, out, layer.workspace(T), logits_in=li, residual=res, flags=flags, logits_out=lo,
                  topk_ids_out=ids)
    st, fl = lib.coli_moe_get_status()
    assert fl == 0, fl
    return bits(out), lo.cpu().numpy(), ids.cpu().numpy()


def _rel_err(got_bits, want_bits):
    got, want = oracle.bf16_bits_to_f64(got_bits), oracle.bf16_bits_to_f64(want_bits)
    assert np.isfinite(got).all()
    return np.abs(got - want).max() / np.abs(want).max()


def test_decode_b64_zipf_every_token(lib):
    shape = synth.DECODE_B64
    li = synth.LayerInputs(shape)
    rw, bias = li.router_w(), li.bias()
    layer = device_layer(shape)
    x = synth.activations(shape)
    out, lo, ids = _gpu_layer(lib, layer, x)
    del layer
    torch.cuda.empty_cache()
    l64, _ = oracle.router_logits(x, rw)
    assert np.all(np.abs(lo - l64) <= logits_tol(x, rw))
    assert np.array_equal(ids, oracle.route(oracle.add_bias(lo, bias), shape.top_k)[0])
    ref, _ = layer_outputs(shape, 0, 0, x, lo, bias=bias)
    err = _rel_err(out, ref)
    print(f"decode b64 zipf, all 64 tokens: union {len(np.unique(ids))}, max rel err {err:.3e}")
    assert err <= OUT_REL_TOL


def _block_edge_tokens(ids, E, k, n_each=2):
    """First and last token of every prefill token block (block j of a segment
    of cnt pairs: [cnt*j/nb, cnt*(j+1)/nb), nb = ceil(cnt/160)) of the n_each
    hottest and n_each coldest experts."""
    unique, seg_off, perm, _ = oracle.batch_union(ids, E)
    cnt = np.diff(seg_off)
    order = np.argsort(cnt, kind="stable")
    toks = set()
    for u in list(order[:n_each]) + list(order[-n_each:]):
        c = int(cnt[u])
        nb = -(-c // 160)
        for j in range(nb):
            s, e = c * j // nb, c * (j + 1) // nb
            toks.add(int(perm[seg_off[u] + s]) // k)
            toks.add(int(perm[seg_off[u] + e - 1]) // k)
    return toks, cnt[order[:n_each]], cnt[order[-n_each:]]


def test_prefill_4096_block_edges_both_forms(lib):
    shape = synth.PREFILL_4096
    li = synth.LayerInputs(shape)
    lg = li.logits()
    x = synth.activations(shape)
    layer = device_layer(synth.DECODE_B1)          # the same layer's weights
    out_p, lo, ids_p = _gpu_layer(lib, layer, x, logits_in=lg)                 # auto: the prefill form
    out_d, _, ids_d = _gpu_layer(lib, layer, x, logits_in=lg, flags=DECODE)
    del layer
    torch.cuda.empty_cache()
    assert lib.coli_moe_ffn_form(lib.dims_for(6144, 2048, 256, 8, 1), 4096) == lib._lib.COLI_FORM_PREFILL
    assert np.array_equal(lo, lg)
    rid = oracle.route(lg, shape.top_k)[0]
    assert np.array_equal(ids_p, rid) and np.array_equal(ids_d, rid)
    toks, cold, hot = _block_edge_tokens(rid, shape.n_experts, shape.top_k)
    toks |= {0, shape.tokens - 1}
    rng = np.random.default_rng(4096)
    while len(toks) < 64:
        toks.add(int(rng.integers(shape.tokens)))
    toks = np.array(sorted(toks))
    ref, _ = layer_outputs(shape, 0, 0, x[toks], lg[toks])
    err_p, err_d = _rel_err(out_p[toks], ref), _rel_err(out_d[toks], ref)
    print(f"prefill 4096, {len(toks)} tokens (coldest experts {cold.tolist()} tokens, hottest {hot.tolist()}): "
          f"prefill form {err_p:.3e}, decode form {err_d:.3e}")
    assert err_p <= OUT_REL_TOL and err_d <= OUT_REL_TOL
    # and the two forms agree over every token
    assert _rel_err(out_p, out_d) <= OUT_REL_TOL


def test_stack16_every_layer_teacher_forced(lib):
    shape = synth.STACK16_B4
    h = synth.activations(shape)
    per_layer = []
    for l in range(shape.layers):
        li = synth.LayerInputs(shape, 0, l)
        layer = device_layer(shape, seed=0, layer=l)
        out, lo, ids = _gpu_layer(lib, layer, h, residual_bits=h, flags=PRENORM)
        del layer
        torch.cuda.empty_cache()
        xin = oracle.rms_norm(h)
        rw = li.router_w()
        l64, _ = oracle.router_logits(xin, rw)
        assert np.all(np.abs(lo - l64) <= logits_tol(xin, rw)), l
        assert np.array_equal(ids, oracle.route(lo, shape.top_k)[0]), l
        per_layer.append((h, lo, out))
        h = out
    refs = layer_jobs([(shape, 0, l, hl, lol, hl, True, None) for l, (hl, lol, _) in enumerate(per_layer)])
    errs = [_rel_err(out, ref) for (_, _, out), ref in zip(per_layer, refs)]
    print("stack 16 x b4, per-layer max rel err: " + " ".join(f"{e:.2e}" for e in errs))
    assert max(errs) <= OUT_REL_TOL


def test_prefill_4096_with_router_logits(lib):
    """The prefill chunk with its router logits computed in the step (the tiled
    fp32 logits kernel at T = 4096, H = 6144): every logit within the derived
    fp32 bound of the oracle's float64 value, routing from those logits bit-exact,
    and 32 tokens of output against the C oracle."""
    shape = synth.PREFILL_4096_ROUTER
    li = synth.LayerInputs(shape)
    rw = li.router_w()
    x = synth.activations(shape)
    layer = device_layer(synth.DECODE_B1)          # the same layer's weights and router
    out, lo, ids = _gpu_layer(lib, layer, x)
    del layer
    torch.cuda.empty_cache()
    l64, _ = oracle.router_logits(x, rw)
    tol = logits_tol(x, rw)
    assert np.all(np.abs(lo - l64) <= tol), np.abs(lo - l64).max()
    assert np.array_equal(ids, oracle.route(lo, shape.top_k)[0])
    toks = np.unique(np.concatenate([[0, shape.tokens - 1], np.random.default_rng(7).integers(0, shape.tokens, 30)]))
    ref, _ = layer_outputs(shape, 0, 0, x[toks], lo[toks])
    err = _rel_err(out[toks], ref)
    xa = np.abs(synth.bf16_bits_to_f32(x).astype(np.float64)) @ np.abs(rw.astype(np.float64)).T
    print(f"prefill 4096 with router logits: {len(toks)} tokens, max rel err {err:.3e}, "
          f"max logit error {np.abs(lo - l64).max():.2e} "
          f"({(np.abs(lo - l64) / (2.0 ** -24 * xa)).max():.2f} x 2^-24 sum|x w|)")
    assert err <= OUT_REL_TOL
