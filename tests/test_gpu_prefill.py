"""Parity of the prefill form of the expert FFN (tcgen05 grouped GEMM) with the
CPU oracle, through the C ABI.

The form is forced with COLI_PATH_PREFILL on shapes the oracle computes in
full: one-stage and multi-stage K, token blocks split near-equally once a
segment passes 160 tokens, experts with a single token, shared experts,
residual and pre-norm.  The full prefill chunk (4096 tokens, 256 experts) is
compared with the C oracle on many tokens in ``tests/test_gpu_fullsize.py``.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._gpu import OUT_REL_TOL, bits, device_layer, needs_gpu, oracle_weights, to_dev_bits
from tests.test_gpu_parity import _small_shape, _status, check_layer, lib, run_gpu_layer  # noqa: F401

pytestmark = [pytest.mark.gpu, needs_gpu]

PREFILL = 0x20   # COLI_PATH_PREFILL
DECODE = 0x10    # COLI_PATH_DECODE


@pytest.mark.parametrize("kw", [
    dict(tokens=64),                                                  # K = 256 / 128: one code stage each
    dict(tokens=33, n_experts=64, top_k=4, n_shared=1),               # many one-token experts
    dict(tokens=200, hidden=512, inter=256, n_experts=8, n_shared=1),  # K = 512: two code stages, 2-D scale maps
    dict(tokens=400, inter=256, n_experts=4, n_shared=1),             # ~200-token segments: two blocks each
    dict(tokens=90, hidden=1024, inter=512, n_experts=6, top_k=3, n_shared=2)],
    ids=lambda kw: "-".join(f"{k}{v}" for k, v in kw.items()))
def test_prefill_form_small_shapes(lib, kw):
    shape = _small_shape(**kw)
    layer = device_layer(shape, seed=7)
    li = synth.LayerInputs(shape, seed=7)
    x = synth.normal_bf16(7, 5, synth.X_IN, (shape.tokens, shape.hidden))
    res = synth.normal_bf16(7, 6, synth.X_IN, (shape.tokens, shape.hidden))
    err, g = check_layer(lib, shape, layer, oracle_weights(shape, seed=7), x, rw=li.router_w(), residual_bits=res,
                         flags=PREFILL)
    print(f"prefill form {shape.tokens} tokens: max rel err {err:.3e}")


def test_prefill_form_hot_expert_and_prenorm(lib):
    """One expert takes all 300 tokens (two blocks of 150); pre-norm layer with residual."""
    shape = _small_shape(tokens=300, n_shared=1)
    layer = device_layer(shape, seed=8)
    rng = np.random.default_rng(8)
    l = rng.standard_normal((300, 16)).astype(np.float32)
    l[:, 3] += 50.0
    x = synth.normal_bf16(8, 5, synth.X_IN, (300, shape.hidden))
    check_layer(lib, shape, layer, oracle_weights(shape, seed=8), x, logits_in=l, flags=PREFILL)
    li = synth.LayerInputs(shape, seed=8)
    check_layer(lib, shape, layer, oracle_weights(shape, seed=8), x, rw=li.router_w(), residual_bits=x,
                flags=PREFILL | lib._lib.COLI_LAYER_PRENORM, max_ambiguous=3)


def _dist_to_exact(lib, shape, layer, W, x, flags):
    """Largest |GPU output - unrounded float64 oracle sum| over max|sum|, with
    the GPU's own routing fed to the oracle (the FFN arithmetic alone)."""
    g = run_gpu_layer(lib, layer, x, flags=flags)
    assert g["flags"] == 0
    _, acc = oracle.moe_ffn_combine(W, x, g["ids"], g["w"], shape.n_experts, shape.n_shared, return_f64=True)
    return np.abs(oracle.bf16_bits_to_f64(g["out"]) - acc).max() / np.abs(acc).max()


def test_prefill_form_arithmetic_error(lib):
    """Distance of each form's output to the oracle's unrounded float64 sum.
    Rounding the output to bf16 alone costs up to 2^-8 of a value (half an ulp
    of an 8-bit significand); the rest is the form's arithmetic, allowed 1e-3
    here.  The prefill form's fp16 operands (each weight q * s rounded once at
    11 bits) keep it at the decode form's level."""
    shape = _small_shape(tokens=96, hidden=1024, inter=512, n_experts=8, top_k=2, n_shared=1)
    layer = device_layer(shape, seed=17)
    W = oracle_weights(shape, seed=17)
    x = synth.normal_bf16(17, 5, synth.X_IN, (96, shape.hidden))
    dp = _dist_to_exact(lib, shape, layer, W, x, PREFILL)
    dd = _dist_to_exact(lib, shape, layer, W, x, DECODE)
    print(f"distance to the unrounded oracle: prefill form {dp:.3e}, decode form {dd:.3e} (2^-8 = {2.0 ** -8:.3e})")
    assert dp <= 2.0 ** -8 + 1e-3 and dd <= 2.0 ** -8 + 1e-3


def test_prefill_form_flags_inputs_fp16_cannot_hold(lib):
    """The prefill form's MMA operands are fp16 copies of the bf16 expert
    input and h: an input of magnitude 65536 or more sets COLI_FLAG_RANGE
    (the call's outputs are undefined); the next call is clean."""
    shape = _small_shape(tokens=40, n_shared=1)
    layer = device_layer(shape, seed=16)
    li = synth.LayerInputs(shape, seed=16)
    x = synth.normal_bf16(16, 5, synth.X_IN, (40, shape.hidden))
    big = x.copy()
    big[3, 17] = 0x47C3          # bf16 99840
    g = run_gpu_layer(lib, layer, big, flags=PREFILL)
    assert g["flags"] & lib._lib.COLI_FLAG_RANGE
    check_layer(lib, shape, layer, oracle_weights(shape, seed=16), x, rw=li.router_w(), flags=PREFILL)
    g = run_gpu_layer(lib, layer, big)          # the decode form holds it
    assert g["flags"] == 0


def test_both_form_flags_are_rejected(lib):
    shape = _small_shape(tokens=40)
    layer = device_layer(shape, seed=9)
    x = to_dev_bits(synth.normal_bf16(9, 5, synth.X_IN, (40, shape.hidden)))
    with pytest.raises(lib.ColiError):
        layer.forward(x, torch.empty_like(x), layer.workspace(40), flags=PREFILL | DECODE)


@pytest.mark.parametrize("T", [1, 3, 8])
def test_prefill_form_at_decode_batch_sizes(lib, T):
    """Tiles of 1..8 tokens (MMA N = 16 with padding columns)."""
    shape = _small_shape(tokens=T, n_shared=1)
    layer = device_layer(shape, seed=12)
    li = synth.LayerInputs(shape, seed=12)
    x = synth.normal_bf16(12, 5, synth.X_IN, (T, shape.hidden))
    check_layer(lib, shape, layer, oracle_weights(shape, seed=12), x, rw=li.router_w(), residual_bits=x,
                flags=PREFILL)


def test_prefill_and_decode_forms_agree_small(lib):
    """Same routed batch through both forms: identical routing, outputs within
    the layer tolerance of each other."""
    shape = _small_shape(tokens=96, hidden=512, inter=256, n_experts=8, n_shared=1)
    layer = device_layer(shape, seed=10)
    li = synth.LayerInputs(shape, seed=10)
    x = synth.normal_bf16(10, 5, synth.X_IN, (96, shape.hidden))
    W = oracle_weights(shape, seed=10)
    _, gp = check_layer(lib, shape, layer, W, x, rw=li.router_w(), flags=PREFILL)
    _, gd = check_layer(lib, shape, layer, W, x, rw=li.router_w(), flags=DECODE)
    assert np.array_equal(gp["ids"], gd["ids"])
    a, b = oracle.bf16_bits_to_f64(gp["out"]), oracle.bf16_bits_to_f64(gd["out"])
    assert np.abs(a - b).max() <= OUT_REL_TOL * np.abs(b).max()


@pytest.fixture(scope="module")
def glm_layer_pf():
    layer = device_layer(synth.DECODE_B1)
    yield layer
    del layer
    torch.cuda.empty_cache()


def test_glm_decode_b1_prefill_form(lib, glm_layer_pf):
    shape = synth.DECODE_B1
    li = synth.LayerInputs(shape)
    err, g = check_layer(lib, shape, glm_layer_pf, oracle_weights(shape), synth.activations(shape),
                         rw=li.router_w(), flags=PREFILL)
    print(f"decode b1 through the prefill form: max rel err {err:.3e}")
