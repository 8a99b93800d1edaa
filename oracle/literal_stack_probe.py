"""Shows why the 16-layer stack needs a normalisation.

Runs the literal stack h_{l+1} = bf16(h_l + MoE_l(h_l)) -- no normalisation --
with the oracle on one GLM-shaped token and prints max|h| and max|MoE(h)|
after each layer (stopping if h stops being finite in bf16).  Calls only
oracle/ and synth/.

    python -m oracle.literal_stack_probe [--layers 6]
"""
import argparse

import numpy as np

import oracle
import synth


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--layers", type=int, default=6)
    a = ap.parse_args()
    shape = synth.STACK16_B4
    h = synth.activations(shape)[:1]
    for l in range(a.layers):
        li = synth.LayerInputs(shape, 0, l)
        W = oracle.ExpertWeights.from_synth(li)
        r = oracle.moe_layer(W, h, shape.n_experts, shape.top_k, shape.n_shared, router_w=li.router_w(),
                             residual_bits=h)
        moe = oracle.moe_ffn_combine(W, h, r["ids"], r["w"], shape.n_experts, shape.n_shared)
        h = r["out"]
        v = oracle.bf16_bits_to_f64(h)
        fin = np.isfinite(v)
        m = oracle.bf16_bits_to_f64(moe)
        print(f"layer {l}: max|h| = {np.abs(v[fin]).max() if fin.any() else float('nan'):.3e}, "
              f"max|MoE(h)| = {np.abs(m).max():.3e}, non-finite {int((~fin).sum())} of {v.size}", flush=True)
        if not fin.all():
            break


if __name__ == "__main__":
    main()
