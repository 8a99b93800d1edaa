"""Parity of the split-K decode form (batches of up to 8 tokens) with the CPU
oracle, through the C ABI.

For T <= 8 (and I a multiple of 256) the layer's FFN is one cooperative
kernel in which each gate/up tile's CTA also computes that tile's K slice of
the down projection for every output row; the partial y's are combined in a
fixed order after a grid-wide wait.  The shapes here cover one and several
down stages, a ragged last down stage (H not a multiple of 512), several
K slices, shared experts, residuals, batches of 1..8 tokens and both
container groups.
"""
import numpy as np
import pytest

import synth
from tests._gpu import device_layer, needs_gpu, oracle_weights
from tests.test_gpu_parity import _small_shape, check_layer, lib, run_gpu_layer  # noqa: F401

pytestmark = [pytest.mark.gpu, needs_gpu]


@pytest.mark.parametrize("kw", [
    dict(tokens=1, inter=256),                                          # 2 K slices, one 256-row down stage
    dict(tokens=3, hidden=768, inter=512, n_shared=1),                  # ragged last down stage (512 + 256 rows)
    dict(tokens=8, hidden=1024, inter=1024, n_experts=8, n_shared=2),   # 8 K slices, two full down stages
    dict(tokens=8, hidden=512, inter=256, n_experts=64, top_k=4),       # 32 pairs on up to 32 experts
    dict(tokens=5, hidden=512, inter=512, group=64, n_shared=1),        # gs64
    dict(tokens=2, hidden=1536, inter=768, n_experts=12, top_k=3)],     # 6 K slices, 3 down stages
    ids=lambda kw: "-".join(f"{k}{v}" for k, v in kw.items()))
def test_splitk_small_shapes(lib, kw):
    shape = _small_shape(**kw)
    layer = device_layer(shape, seed=31)
    li = synth.LayerInputs(shape, seed=31)
    x = synth.normal_bf16(31, 5, synth.X_IN, (shape.tokens, shape.hidden))
    res = synth.normal_bf16(31, 6, synth.X_IN, (shape.tokens, shape.hidden))
    err, g = check_layer(lib, shape, layer, oracle_weights(shape, seed=31), x, rw=li.router_w(), residual_bits=res)
    print(f"split-K {kw}: max rel err {err:.3e}")


def test_splitk_batch_invariance_small(lib):
    """Each token of an 8-token batch gives the bits it gives alone."""
    shape = _small_shape(tokens=8, hidden=768, inter=512, n_experts=16, top_k=2, n_shared=1)
    layer = device_layer(shape, seed=32)
    x = synth.normal_bf16(32, 5, synth.X_IN, (8, shape.hidden))
    gb = run_gpu_layer(lib, layer, x, residual_bits=x)
    assert gb["flags"] == 0
    for t in range(8):
        g1 = run_gpu_layer(lib, layer, x[t:t + 1], residual_bits=x[t:t + 1])
        assert np.array_equal(g1["ids"][0], gb["ids"][t])
        assert np.array_equal(g1["out"][0], gb["out"][t]), t
