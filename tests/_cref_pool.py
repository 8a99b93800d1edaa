"""The plain-C oracle on many tokens of a full-size layer, over the host's
cores -- test infrastructure for the GPU parity tests.

Each token is one C-oracle call on that token alone (the layer's output for a
token depends on no other token), with the weights of only the experts it
selects regenerated from the seeded generator.  The calls are spread over a
pool of spawned processes (never forked: the parent holds a CUDA context).
Routing is fed from given fp32 logits (the GPU's own, or the workload's), so
that both sides route from the same numbers.
"""
from __future__ import annotations

import os

import numpy as np

import synth

_KINDS = {"gate": (synth.GATE_Q, synth.GATE_S), "up": (synth.UP_Q, synth.UP_S), "down": (synth.DOWN_Q, synth.DOWN_S)}
_cache: dict = {}


def _fetch(shape, seed, layer, kind, e):
    key = (shape.name, seed, layer, kind, e)
    if key not in _cache:
        if len(_cache) > 96:
            _cache.clear()
        li = synth.LayerInputs(shape, seed, layer)
        q, s = _KINDS[kind]
        _cache[key] = (li.expert_codes(q, e), li.expert_scales(s, e))
    return _cache[key]


def _work(shape, seed, layer, x, logits, residual, prenorm, bias):
    import oracle.cref as cr
    cr.build()
    outs, accs = [], []
    for t in range(x.shape[0]):
        xt = x[t:t + 1]
        xin = cr.rms_norm(xt) if prenorm else xt
        r = cr.moe_layer_experts(lambda kind, e: _fetch(shape, seed, layer, kind, e), shape.hidden, shape.inter,
                                 xin, shape.n_experts, shape.top_k, shape.n_shared, shape.group, shape.bits,
                                 bias=bias, logits_in=logits[t:t + 1],
                                 residual_bits=None if residual is None else residual[t:t + 1])
        outs.append(r["out"][0])
        accs.append(r["acc"][0])
    return np.stack(outs), np.stack(accs)


def layer_outputs(shape, seed: int, layer: int, x_bits, logits, residual_bits=None, prenorm: bool = False,
                  bias=None, procs: int | None = None):
    """C-oracle outputs (bf16 bits [n, H]) and their float64 sums of the layer
    on the rows of x_bits, routed from `logits` (fp32 [n, E]) plus `bias`."""
    import multiprocessing as mp
    n = x_bits.shape[0]
    procs = max(1, min(procs or os.cpu_count() or 1, n))
    parts = np.array_split(np.arange(n), procs)
    args = [(shape, seed, layer, np.ascontiguousarray(x_bits[p]), np.ascontiguousarray(logits[p]),
             None if residual_bits is None else np.ascontiguousarray(residual_bits[p]), prenorm, bias)
            for p in parts if len(p)]
    with mp.get_context("spawn").Pool(len(args)) as pool:
        res = pool.starmap(_work, args)
    return np.concatenate([r[0] for r in res]), np.concatenate([r[1] for r in res])


def layer_jobs(jobs, procs: int | None = None):
    """Several layers' tokens in one pool: jobs = [(shape, seed, layer, x_bits,
    logits, residual_bits or None, prenorm, bias)], one row per token each.
    Returns the C-oracle output rows (bf16 bits) of each job."""
    import multiprocessing as mp
    units = []      # (job, rows) split so that every process gets work
    total = sum(j[3].shape[0] for j in jobs)
    procs = max(1, min(procs or os.cpu_count() or 1, total))
    per = -(-total // procs)
    for ji, (shape, seed, layer, x, lg, res, pn, bias) in enumerate(jobs):
        for r0 in range(0, x.shape[0], per):
            rows = np.arange(r0, min(x.shape[0], r0 + per))
            units.append((ji, rows, (shape, seed, layer, np.ascontiguousarray(x[rows]), np.ascontiguousarray(lg[rows]),
                                     None if res is None else np.ascontiguousarray(res[rows]), pn, bias)))
    with mp.get_context("spawn").Pool(min(procs, len(units))) as pool:
        res = pool.starmap(_work, [u[2] for u in units])
    outs = [np.empty((j[3].shape[0], j[0].hidden), np.uint16) for j in jobs]
    for (ji, rows, _), (o, _) in zip(units, res):
        outs[ji][rows] = o
    return outs
