"""The allocation-free layer call matches the workspace one.

coli_moe_layer_noalloc is for callers that cannot allocate device memory
while they run the layer -- for example a plugin inside another runtime that
owns every device allocation, or a real-time loop whose memory is fixed up
front.  It uses scratch that the library keeps in device memory instead of a
caller workspace.  These tests call it through the C ABI twice in a row, with
different inputs, and compare each result with coli_moe_layer's on the same
inputs: within the layer's output tolerance, and bit for bit, since the two
run the same kernels on the same data and scratch left over from an earlier
call must change nothing.  A third call with a larger batch, which takes
another FFN form, checks the same after the shared scratch was last used by
a different form.  This file is collected last.
"""
import numpy as np
import pytest
import torch

import synth
from tests._gpu import OUT_REL_TOL, bits, device_layer, needs_gpu, to_dev_bits

pytestmark = [pytest.mark.gpu, needs_gpu]


def _both(m, layer, x_bits, residual_bits=None, flags=0):
    T = x_bits.shape[0]
    d = layer.dims
    x = to_dev_bits(x_bits)
    res = None if residual_bits is None else to_dev_bits(residual_bits)
    out_ws, out_na = torch.empty_like(x), torch.empty_like(x)
    ids_ws = torch.empty((T, d.top_k), dtype=torch.int32, device="cuda")
    ids_na = torch.empty_like(ids_ws)
    layer.forward(x, out_ws, layer.workspace(T), residual=res, flags=flags, topk_ids_out=ids_ws)
    m.coli_moe_layer_noalloc(d, layer.weights, x, out_na, residual=res, flags=flags, topk_ids_out=ids_na)
    st, fl = m.coli_moe_get_status()
    assert st == 0 and fl == 0
    return bits(out_ws), bits(out_na), ids_ws.cpu().numpy(), ids_na.cpu().numpy()


def _close(a_bits, b_bits):
    import oracle
    a, b = oracle.bf16_bits_to_f64(a_bits), oracle.bf16_bits_to_f64(b_bits)
    return np.abs(a - b).max() <= OUT_REL_TOL * np.abs(a).max()


def test_noalloc_matches_workspace_call_glm_decode():
    import int4_routed_expert_renorm_b200 as m
    shape = synth.DECODE_B1
    layer = device_layer(shape)
    # two batch-1 calls in a row (split-K form), then 9 tokens (two-phase form)
    for batch, T in ((0, 1), (1, 1), (2, 9)):
        x = np.concatenate([synth.activations(shape, 0, 10 * batch + t) for t in range(T)])
        o_ws, o_na, i_ws, i_na = _both(m, layer, x)
        assert np.array_equal(i_ws, i_na)
        assert _close(o_ws, o_na)
        assert np.array_equal(o_ws, o_na)
    del layer
    torch.cuda.empty_cache()


def test_noalloc_matches_workspace_call_prenorm_residual():
    import int4_routed_expert_renorm_b200 as m
    shape = synth.LayerShape("small", 256, 128, 16, 2, 1, 5)
    layer = device_layer(shape, seed=7)
    for batch, T in ((0, 5), (1, 5), (2, 40)):
        x = synth.normal_bf16(7, batch, synth.X_IN, (T, 256))
        o_ws, o_na, i_ws, i_na = _both(m, layer, x, residual_bits=x, flags=m._lib.COLI_LAYER_PRENORM)
        assert np.array_equal(i_ws, i_na)
        assert _close(o_ws, o_na)
        assert np.array_equal(o_ws, o_na)


def test_noalloc_rejects_batches_beyond_its_scratch():
    import int4_routed_expert_renorm_b200 as m
    shape = synth.LayerShape("small", 256, 128, 16, 2, 1, 4)
    layer = device_layer(shape, seed=8)
    T = 1
    while m.coli_moe_workspace_bytes(layer.dims, T) <= m._lib.COLI_NOALLOC_SCRATCH_BYTES:
        T *= 2
    x = torch.zeros((T, 256), dtype=torch.int16, device="cuda")
    with pytest.raises(m.ColiError) as e:
        m.coli_moe_layer_noalloc(layer.dims, layer.weights, x, torch.empty_like(x))
    assert e.value.status == m._lib.COLI_ERR_WORKSPACE
