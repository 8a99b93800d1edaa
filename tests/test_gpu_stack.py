"""The 16-layer stack (decode batch 4, residual add and pre-norm between
layers) against the oracle, through the C ABI.

Every layer is checked on the GPU's own hidden state: the oracle normalises
it, routes from its own logits and runs the layer, and the GPU layer output
must match within the layer tolerance (routing bit-exact outside near-ties).
On the reduced shape the oracle also runs the whole chain from the same
input, and the final hidden states are compared, within the same 1e-2 of the
largest magnitude.  Every layer of the GLM-5.2-shaped stack is checked in
``tests/test_gpu_fullsize.py``.
"""
import numpy as np
import pytest

import oracle
import synth
from tests._gpu import OUT_REL_TOL, device_layer, needs_gpu, oracle_weights
from tests.test_gpu_parity import _small_shape, check_layer, lib  # noqa: F401

pytestmark = [pytest.mark.gpu, needs_gpu]

PRENORM = 0x1


def test_stack16_reduced_shape(lib):
    L = 16
    shape = _small_shape(tokens=4, n_shared=1, layers=L, prenorm=True)
    h0 = synth.normal_bf16(11, 5, synth.X_IN, (4, shape.hidden))
    h = h0
    oracle_layers = []
    for l in range(L):
        layer = device_layer(shape, seed=11, layer=l)
        li = synth.LayerInputs(shape, 11, l)
        W = oracle_weights(shape, seed=11, layer=l)
        oracle_layers.append((W, li.router_w(), None))
        err, g = check_layer(lib, shape, layer, W, h, rw=li.router_w(), residual_bits=h, flags=PRENORM)
        h = g["out"]
    hN, per = oracle.moe_stack(oracle_layers, h0, shape.n_experts, shape.top_k, shape.n_shared)
    got, want = oracle.bf16_bits_to_f64(h), oracle.bf16_bits_to_f64(hN)
    err = np.abs(got - want).max() / np.abs(want).max()
    print(f"stack of {L} (reduced shape): final hidden state max rel err {err:.3e}")
    assert np.isfinite(got).all()
    assert err <= OUT_REL_TOL
