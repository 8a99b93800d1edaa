"""The CUDA layer against the plain-C oracle (oracle/c/moe_ref.c).

The same bars as the numpy-oracle parity tests: router logits within the
derived fp32 bound, expert ids identical and weights within (k + 4) * 2^-22
when both route from the GPU's own fp32 logits (so that a near tie decided by
summation order cannot differ), and max|gpu - ref| <= 1e-2 * max|ref| on the
layer output.  The C oracle reads only the experts the batch selects.
"""
import numpy as np
import pytest

import oracle.cref as cr
import synth
from tests._gpu import OUT_REL_TOL, device_layer, logits_tol, needs_gpu, route_w_tol
from tests.test_gpu_parity import _small_shape, lib, run_gpu_layer  # noqa: F401

pytestmark = [pytest.mark.gpu, needs_gpu]

KINDS = {"gate": (synth.GATE_Q, synth.GATE_S), "up": (synth.UP_Q, synth.UP_S), "down": (synth.DOWN_Q, synth.DOWN_S)}


def c_oracle_check(lib, shape, g, x_bits, seed=0, residual_bits=None, prenorm=False, logits_given=None):
    """Compare one GPU layer result ``g`` (run_gpu_layer) with the C oracle;
    returns the observed relative output error."""
    li = synth.LayerInputs(shape, seed)
    assert g["flags"] == 0, g["flags"]
    xin = cr.rms_norm(x_bits) if prenorm else x_bits
    if logits_given is None:
        l64, _ = cr.router_logits(xin, li.router_w())
        assert np.all(np.abs(g["logits"] - l64) <= logits_tol(xin, li.router_w()))
    else:
        assert np.array_equal(g["logits"], logits_given)
    ref = cr.moe_layer_experts(lambda kind, e: (li.expert_codes(KINDS[kind][0], e), li.expert_scales(KINDS[kind][1], e)),
                               shape.hidden, shape.inter, xin, shape.n_experts, shape.top_k, shape.n_shared,
                               shape.group, shape.bits, logits_in=g["logits"], bias=li.bias(),
                               residual_bits=residual_bits)
    assert not ref["flags"].any()
    assert np.array_equal(g["ids"], ref["ids"])
    assert np.abs(g["w"] - ref["w"]).max(initial=0) <= route_w_tol(shape.top_k)
    got = cr.decode_bf16(g["out"])
    want = cr.decode_bf16(ref["out"])
    assert np.isfinite(got).all()
    err = np.abs(got - want).max() / np.abs(want).max()
    assert err <= OUT_REL_TOL, err
    return err


CASES = [  # (shape kwargs, flags, with residual, given logits)
    (dict(tokens=4), 0, False, False),                                                   # two-phase form, I = 128
    (dict(tokens=3, hidden=768, inter=512, n_shared=1), 0, True, False),                 # split-K form
    (dict(tokens=8, hidden=512, inter=256, n_experts=64, top_k=4), 0, True, False),      # split-K, 32 pairs
    (dict(tokens=5, hidden=512, inter=512, group=64, n_shared=1, bits=8), 0, True, False),   # int8, gs64
    (dict(tokens=20, hidden=512, inter=256, n_experts=8, n_shared=1), 0, True, False),   # two-phase, 16-token blocks
    (dict(tokens=70, hidden=512, inter=256, n_experts=8, n_shared=1), 0, False, True),   # two-phase, 32-token blocks
    (dict(tokens=40, hidden=512, inter=256, n_experts=8, n_shared=1), 0x20, True, True),  # prefill form (forced)
    # pre-norm + residual; logits given, so that a bf16 rounding of the normalised
    # input that fp32 and double decide differently cannot move a logit past the bound
    (dict(tokens=4, hidden=512, inter=256, n_experts=16, n_shared=1), 0x1, True, True),
]


@pytest.mark.parametrize("kw,flags,with_res,given", CASES,
                         ids=lambda v: "-".join(f"{a}{b}" for a, b in v.items()) if isinstance(v, dict) else str(v))
def test_layer_matches_c_oracle(lib, kw, flags, with_res, given):
    shape = _small_shape(**kw)
    layer = device_layer(shape, seed=51)
    T = shape.tokens
    x = synth.normal_bf16(51, 5, synth.X_IN, (T, shape.hidden))
    res = synth.normal_bf16(51, 6, synth.X_IN, (T, shape.hidden)) if with_res else None
    lg = np.random.default_rng(51).standard_normal((T, shape.n_experts)).astype(np.float32) if given else None
    g = run_gpu_layer(lib, layer, x, logits_in=lg, residual_bits=res, flags=flags)
    err = c_oracle_check(lib, shape, g, x, seed=51, residual_bits=res, prenorm=bool(flags & 0x1), logits_given=lg)
    print(f"C oracle {kw} flags {flags:#x}: max rel err {err:.3e}")


@pytest.mark.slow
def test_glm_decode_b1_matches_c_oracle(lib):
    """One token of the GLM-shaped layer (H 6144, I 2048, 256 experts, k 8, one
    shared expert), the split-K decode form, with a residual."""
    shape = synth.DECODE_B1
    layer = device_layer(shape)
    x = synth.activations(shape)
    g = run_gpu_layer(lib, layer, x, residual_bits=x)
    err = c_oracle_check(lib, shape, g, x, residual_bits=x)
    print(f"C oracle, GLM decode b1: max rel err {err:.3e}")
