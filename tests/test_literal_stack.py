"""Why the 16-layer stack carries a weightless pre-norm, pinned.

Taken literally -- h_{l+1} = bf16(h_l + MoE_l(h_l)), with no normalisation --
the stack of GLM-shaped layers with the stated weight and input
distributions does not stay a usable model: the hidden state grows by
orders of magnitude in two layers, after which every gate projection of
every selected expert is negative (codes uniform on [-8, 7] have mean -0.5,
so a hidden state with a large common component drives all of g below 0)
and the MoE output is exactly zero from then on.  The C oracle runs three
layers of the literal stack on one token, reading only the experts the token
selects.  CPU only.
"""
import numpy as np

import oracle
import oracle.cref as cr
import synth

KINDS = {"gate": (synth.GATE_Q, synth.GATE_S), "up": (synth.UP_Q, synth.UP_S), "down": (synth.DOWN_Q, synth.DOWN_S)}


def _layer(shape, l, h, residual):
    li = synth.LayerInputs(shape, 0, l)
    fetch = lambda kind, e: (li.expert_codes(KINDS[kind][0], e), li.expert_scales(KINDS[kind][1], e))  # noqa: E731
    return cr.moe_layer_experts(fetch, shape.hidden, shape.inter, h, shape.n_experts, shape.top_k, shape.n_shared,
                                shape.group, shape.bits, router_w=li.router_w(),
                                residual_bits=h if residual else None)


def test_literal_stack_degenerates():
    cr.build()
    shape = synth.STACK16_B4
    h = synth.activations(shape)[:1]
    growth, moe_max = [], []
    for l in range(3):
        moe = oracle.bf16_bits_to_f64(_layer(shape, l, h, residual=False)["out"])
        h = _layer(shape, l, h, residual=True)["out"]
        v = oracle.bf16_bits_to_f64(h)
        assert np.isfinite(v).all()
        growth.append(np.abs(v).max())
        moe_max.append(np.abs(moe).max())
    # the hidden state (max |x| about 4 at the input) grows by orders of
    # magnitude over the first two layers
    assert growth[0] > 100 and growth[1] > 1e5
    # then the layer contributes nothing at all: every selected gate is negative
    assert moe_max[0] > 0 and moe_max[2] == 0.0
