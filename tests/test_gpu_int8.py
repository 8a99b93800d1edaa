"""Parity of the int8 code container with the CPU oracle, through the C ABI.

The README requires the MTP head to be int8 ("Decodifica speculativa,
onestamente"); the library takes the int4 container with one
two's-complement byte per code (dims.code_bits = 8) through the split-K
decode form: the head's draft batches of up to 8 tokens in one pass, larger
batches in consecutive 8-token passes.  Each code is
split into a signed high nibble (decoded straight to 16 * hi) and an
unsigned low nibble that meet the same activation fragment in the MMA.
"""
import numpy as np
import pytest
import torch

import synth
from tests._gpu import device_layer, needs_gpu, oracle_weights, to_dev_bits
from tests.test_gpu_parity import _small_shape, check_layer, lib, run_gpu_layer  # noqa: F401

pytestmark = [pytest.mark.gpu, needs_gpu]


@pytest.mark.parametrize("kw", [
    dict(tokens=1, inter=256),
    dict(tokens=3, hidden=768, inter=512, n_shared=1),
    dict(tokens=8, hidden=1024, inter=1024, n_experts=8, n_shared=2),
    dict(tokens=8, hidden=512, inter=256, n_experts=64, top_k=4),
    dict(tokens=5, hidden=512, inter=512, group=64, n_shared=1),
    dict(tokens=2, hidden=1536, inter=768, n_experts=12, top_k=3)],
    ids=lambda kw: "-".join(f"{k}{v}" for k, v in kw.items()))
def test_int8_small_shapes(lib, kw):
    shape = _small_shape(bits=8, **kw)
    layer = device_layer(shape, seed=41)
    li = synth.LayerInputs(shape, seed=41)
    x = synth.normal_bf16(41, 5, synth.X_IN, (shape.tokens, shape.hidden))
    res = synth.normal_bf16(41, 6, synth.X_IN, (shape.tokens, shape.hidden))
    err, g = check_layer(lib, shape, layer, oracle_weights(shape, seed=41), x, rw=li.router_w(), residual_bits=res)
    print(f"int8 {kw}: max rel err {err:.3e}")


@pytest.mark.parametrize("T", [9, 20])
def test_int8_batches_above_8_tokens_run_in_passes(lib, T):
    """int8 batches above 8 tokens run as consecutive 8-token split-K passes:
    every token's output is the bits of its own batch-1 output, and the layer
    matches the oracle; the prefill form stays unsupported for int8 codes."""
    shape = _small_shape(bits=8, tokens=T, inter=256)
    layer = device_layer(shape, seed=42)
    li = synth.LayerInputs(shape, seed=42)
    x = synth.normal_bf16(42, 5, synth.X_IN, (T, shape.hidden))
    res = synth.normal_bf16(42, 6, synth.X_IN, (T, shape.hidden))
    err, g = check_layer(lib, shape, layer, oracle_weights(shape, seed=42), x, rw=li.router_w(), residual_bits=res)
    print(f"int8 T={T} in 8-token passes: max rel err {err:.3e}")
    xd, rd = to_dev_bits(x), to_dev_bits(res)
    whole = torch.empty_like(xd)
    layer.forward(xd, whole, layer.workspace(T), residual=rd)
    one = torch.empty_like(xd[:1])
    ws1 = layer.workspace(1)
    for t in range(T):
        layer.forward(xd[t:t + 1].contiguous(), one, ws1, residual=rd[t:t + 1].contiguous())
        assert torch.equal(one[0], whole[t]), t
    st, fl = lib.coli_moe_get_status()
    assert st == 0 and fl == 0
    x4 = xd[:4].contiguous()
    with pytest.raises(lib.ColiError):
        layer.forward(x4, torch.empty_like(x4), layer.workspace(4), flags=0x20)   # COLI_PATH_PREFILL


@pytest.fixture(scope="module")
def glm_int8():
    torch.cuda.empty_cache()
    layer = device_layer(synth.DECODE_B1_INT8)
    yield layer
    del layer
    torch.cuda.empty_cache()


def test_glm_int8_decode_b1_full(lib, glm_int8):
    shape = synth.DECODE_B1_INT8
    li = synth.LayerInputs(shape)
    err, g = check_layer(lib, shape, glm_int8, oracle_weights(shape), synth.activations(shape), rw=li.router_w())
    print(f"int8 decode b1: max rel err {err:.3e}")


def test_glm_int8_batch_invariance(lib, glm_int8):
    """A 4-token draft batch gives each token the bits it gets alone."""
    shape = synth.DECODE_B1_INT8
    x = np.concatenate([synth.activations(shape, 0, b) for b in range(4)])
    gb = run_gpu_layer(lib, glm_int8, x, residual_bits=x, flags=lib._lib.COLI_LAYER_PRENORM)
    assert gb["flags"] == 0
    for t in range(4):
        g1 = run_gpu_layer(lib, glm_int8, x[t:t + 1], residual_bits=x[t:t + 1], flags=lib._lib.COLI_LAYER_PRENORM)
        assert np.array_equal(g1["ids"][0], gb["ids"][t])
        assert np.array_equal(g1["out"][0], gb["out"][t]), t
