"""Bit-exact parity of the batch-union that coli_moe_layer itself computes.

The layer does not call coli_moe_union: batches of 2 to 8 tokens (T*k <=
128, E <= 256) are routed and united by every CTA of the split-K kernel
itself (CTA 0 writes the results out), other small batches in one warp of a
routing kernel (T*k <= 32 and <= 128 take two different sorts), batches up
to 128 tokens in one CTA, larger decode batches in the route + union
kernels, and prefill batches in a many-CTA counting sort.  Each of these
leaves its
unique ids, segment offsets, permutation and inverse in the call's workspace
(coli_moe_union_offsets says where); they are compared element by element
with the oracle's union of the ids the layer selected, and those ids with
the oracle's routing of the same fp32 logits.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._gpu import device_layer, needs_gpu, route_w_tol, to_dev_bits

pytestmark = [pytest.mark.gpu, needs_gpu]


@pytest.fixture(scope="module")
def lib():
    import int4_routed_expert_renorm_b200 as m
    m.coli_moe_get_status()
    return m


def _shape(T, E, k, H=256, I=256, S=1):
    return synth.LayerShape(f"union_t{T}_e{E}_k{k}", H, I, E, k, S, T)


# (T, E, k, logits kind, the union code the layer runs for it)
CASES = [
    (1, 256, 8, "normal", "routing kernel, one warp, T*k <= 32"),
    (4, 256, 8, "normal", "split-K kernel's own routing, T*k <= 32"),
    (8, 256, 8, "zipf", "split-K kernel's own routing, T*k <= 128"),
    (3, 16, 2, "ties", "split-K kernel's own routing, tie-dense logits"),
    (6, 200, 4, "normal", "split-K kernel's own routing, E not a multiple of 32"),
    (4, 512, 8, "normal", "routing kernel for E > 256, split-K form"),
    (8, 64, 32, "ties", "one CTA for T*k > 128, split-K form"),
    (16, 256, 8, "zipf", "one warp, T*k <= 128"),
    (11, 16, 2, "ties", "one warp, T*k <= 32, tie-dense logits"),
    (17, 256, 8, "normal", "one CTA, T <= 128"),
    (128, 64, 8, "ties", "one CTA, T <= 128, tie-dense logits"),
    (200, 256, 8, "zipf", "route + union kernels"),
    (4096, 256, 8, "normal", "many-CTA union (prefill form)"),
]


@pytest.mark.parametrize("T,E,k,kind,path", CASES, ids=[f"T{c[0]}-E{c[1]}-k{c[2]}-{c[3]}" for c in CASES])
def test_layer_union_bit_exact(lib, T, E, k, kind, path):
    shape = _shape(T, E, k)
    layer = device_layer(shape, seed=21)
    rng = np.random.default_rng(T * 131 + E)
    if kind == "ties":
        l32 = rng.integers(0, 4, size=(T, E)).astype(np.float32)
    else:
        l32 = rng.standard_normal((T, E)).astype(np.float32)
    if kind == "zipf":
        l32 += synth.zipf_bias(0, 0, E)
    x = synth.normal_bf16(21, 5, synth.X_IN, (T, shape.hidden))
    xd = to_dev_bits(x)
    out = torch.empty_like(xd)
    ws = layer.workspace(T)
    ws.fill_(0x5A)                                 # whatever the workspace held before
    ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    layer.forward(xd, out, ws, logits_in=torch.from_numpy(l32).cuda(), topk_ids_out=ids, topk_w_out=w)
    st, flags = lib.coli_moe_get_status()
    assert flags == 0
    rid, rw, rfl = oracle.route(l32, k)
    gid = ids.cpu().numpy()
    assert np.array_equal(gid, rid)
    assert np.abs(w.cpu().numpy() - rw).max() <= route_w_tol(k)
    off = lib.coli_moe_union_offsets(layer.dims, T)
    P, Umax = T * k, min(E, T * k)
    wsn = ws.cpu().numpy()

    def i32(o, n):
        return wsn[o:o + 4 * n].view(np.int32)

    ru, rs, rp, rpp = oracle.batch_union(rid, E)
    U = int(i32(off[1], 1)[0])
    assert U == len(ru) and U <= Umax
    assert np.array_equal(i32(off[0], U), ru)
    assert np.array_equal(i32(off[2], U + 1), rs)
    assert np.array_equal(i32(off[3], P), rp)
    assert np.array_equal(i32(off[4], P), rpp)


def test_union_offsets_lie_inside_the_workspace(lib):
    """The five regions are disjoint, 4-byte aligned and inside the bytes a
    call of T tokens needs."""
    for T, E, k in ((1, 256, 8), (64, 256, 8), (4096, 256, 8), (3, 16, 2)):
        dims = lib.dims_for(256, 256, E, k, 1)
        off = lib.coli_moe_union_offsets(dims, T)
        sizes = [min(E, T * k), 1, min(E, T * k) + 1, T * k, T * k]
        spans = sorted((o, o + 4 * n) for o, n in zip(off, sizes))
        assert all(o % 4 == 0 for o in off)
        assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))
        assert spans[-1][1] <= lib.coli_moe_workspace_bytes(dims, T)


@pytest.mark.parametrize("T", [1, 6], ids=["routing-kernel", "split-K-own-routing"])
def test_layer_nonfinite_logits_flagged(lib, T):
    """NaN and +inf logits set COLI_FLAG_NONFINITE on the layer path too, and
    the selection stays the oracle's (NaN ranks as -inf)."""
    E, k = 32, 4
    shape = _shape(T, E, k)
    layer = device_layer(shape, seed=22)
    l32 = np.random.default_rng(5 + T).standard_normal((T, E)).astype(np.float32)
    l32[0, 5] = np.nan
    l32[T - 1, 0] = np.inf
    x = synth.normal_bf16(22, 5, synth.X_IN, (T, shape.hidden))
    xd = to_dev_bits(x)
    out = torch.empty_like(xd)
    ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
    lib.coli_moe_get_status()                      # clears the flags
    layer.forward(xd, out, layer.workspace(T), logits_in=torch.from_numpy(l32).cuda(), topk_ids_out=ids)
    st, flags = lib.coli_moe_get_status()
    assert flags & lib._lib.COLI_FLAG_NONFINITE
    assert np.array_equal(ids.cpu().numpy(), oracle.route(l32, k)[0])
