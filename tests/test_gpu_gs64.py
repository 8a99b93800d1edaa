"""Parity of the group-64 ("gs64") container with the CPU oracle, through the
C ABI.

The gs64 container (Colibri README, "2. Scarica il modello") stores one fp16
scale per 64 codes along K instead of one per 32.  Both FFN forms read it: the
decode form (mma.sync, 512-K down stages for T <= 8, 256-K stages above) and
the prefill form (tcgen05).  Besides the oracle, every form is checked against
the group-32 container whose two scales of every 64-wide span are that span's
scale: both describe the same weights, and the kernels scale each 32-wide
partial sum by its scale in the same order, so the outputs are bit-identical.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._gpu import OUT_REL_TOL, device_layer, needs_gpu, oracle_weights
from tests.test_gpu_parity import _small_shape, check_layer, lib, run_gpu_layer  # noqa: F401

pytestmark = [pytest.mark.gpu, needs_gpu]

PREFILL = 0x20   # COLI_PATH_PREFILL
DECODE = 0x10    # COLI_PATH_DECODE
FORMS = {"decode": DECODE, "prefill": PREFILL}


def _as_group32(layer):
    """The same weights in the group-32 container (every scale repeated twice)."""
    from int4_routed_expert_renorm_b200 import MoELayer, dims_for
    d = layer.dims
    t = dict(layer.t)
    for name in ("gate_s", "up_s", "down_s"):
        t[name] = torch.repeat_interleave(layer.t[name], 2, dim=-1).contiguous()
    dims = dims_for(d.hidden, d.inter, d.n_experts, d.top_k, d.n_shared, 32)
    return MoELayer(dims, t, layer.router_w, layer.bias)


def test_device_fill_gs64_matches_numpy_generator():
    import synth.gpu as sg
    shape = synth.DECODE_B1_GS64
    t = sg.expert_tensors(shape)
    li = synth.LayerInputs(shape)
    assert t["gate_s"].shape == (shape.n_total, shape.inter, shape.hidden // 64)
    for e in (0, 200, shape.n_total - 1):
        for name, sk in (("gate", synth.GATE_S), ("up", synth.UP_S), ("down", synth.DOWN_S)):
            assert np.array_equal(t[name + "_s"][e].cpu().numpy().view(np.uint16), li.expert_scales(sk, e))
    del t
    torch.cuda.empty_cache()


@pytest.mark.parametrize("form", ["decode", "prefill"])
@pytest.mark.parametrize("kw", [
    dict(tokens=1, hidden=512, inter=512, n_shared=1),                 # down K = 512: one stage, 1-D scale copy
    dict(tokens=6, hidden=1024, inter=1024, n_experts=8, n_shared=1),   # two 512-K down stages
    dict(tokens=40, hidden=512, inter=512, top_k=4, n_shared=1),        # 32-token tiles, 256-K stages
    dict(tokens=200, hidden=1024, inter=512, n_experts=8, n_shared=2)],
    ids=lambda kw: "-".join(f"{k}{v}" for k, v in kw.items()))
def test_gs64_small_shapes(lib, kw, form):
    shape = _small_shape(group=64, **kw)
    layer = device_layer(shape, seed=21)
    li = synth.LayerInputs(shape, seed=21)
    x = synth.normal_bf16(21, 5, synth.X_IN, (shape.tokens, shape.hidden))
    res = synth.normal_bf16(21, 6, synth.X_IN, (shape.tokens, shape.hidden))
    err, g = check_layer(lib, shape, layer, oracle_weights(shape, seed=21), x, rw=li.router_w(), residual_bits=res,
                         flags=FORMS[form])
    print(f"gs64 {form} form, {shape.tokens} tokens: max rel err {err:.3e}")
    g32 = run_gpu_layer(lib, _as_group32(layer), x, residual_bits=res, flags=FORMS[form])
    assert g32["flags"] == 0
    assert np.array_equal(g32["ids"], g["ids"])
    assert np.array_equal(g32["out"], g["out"])


@pytest.fixture(scope="module")
def glm_gs64():
    torch.cuda.empty_cache()
    layer = device_layer(synth.DECODE_B1_GS64)
    yield layer
    del layer
    torch.cuda.empty_cache()


@pytest.mark.parametrize("form", ["decode", "prefill"])
def test_glm_gs64_decode_b1_full(lib, glm_gs64, form):
    shape = synth.DECODE_B1_GS64
    li = synth.LayerInputs(shape)
    err, g = check_layer(lib, shape, glm_gs64, oracle_weights(shape), synth.activations(shape), rw=li.router_w(),
                         flags=FORMS[form])
    print(f"gs64 decode b1 ({form} form): max rel err {err:.3e}")


def test_glm_gs64_prefill_4096(lib, glm_gs64):
    """Sampled tokens against the oracle; every token of the prefill form
    against the decode form."""
    shape = synth.PREFILL_4096_GS64
    li = synth.LayerInputs(shape)
    x = synth.activations(shape)
    lg = li.logits()
    err, gp = check_layer(lib, shape, glm_gs64, oracle_weights(shape), x, sample=[0, 9, 2047, 4095], logits_in=lg,
                          flags=PREFILL)
    gd = run_gpu_layer(lib, glm_gs64, x, logits_in=lg, flags=DECODE)
    assert gd["flags"] == 0
    assert np.array_equal(gp["ids"], gd["ids"])
    a, b = oracle.bf16_bits_to_f64(gp["out"]), oracle.bf16_bits_to_f64(gd["out"])
    diff = np.abs(a - b).max() / np.abs(b).max()
    print(f"gs64 prefill 4096: sampled max rel err {err:.3e}; prefill vs decode form {diff:.3e}")
    assert diff <= OUT_REL_TOL


def test_glm_gs64_batch_invariance(lib, glm_gs64):
    shape = synth.DECODE_B1_GS64
    T = 4
    x = np.concatenate([synth.activations(shape, 0, b) for b in range(T)])
    gb = run_gpu_layer(lib, glm_gs64, x)
    assert gb["flags"] == 0
    for t in range(T):
        g1 = run_gpu_layer(lib, glm_gs64, x[t:t + 1])
        assert np.array_equal(g1["ids"][0], gb["ids"][t])
        assert np.array_equal(g1["out"][0], gb["out"][t]), t
