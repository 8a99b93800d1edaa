"""Bit-exact parity of the batch-union that coli_moe_layer itself computes.

The layer does not call coli_moe_union: small batches route and unite in one
warp (T*k <= 32 and <= 128 take two different sorts), batches up to 128
tokens in one CTA, larger decode batches in the route + union kernels, and
prefill batches in a many-CTA counting sort.  Each of these leaves its
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
    (1, 256, 8, "normal", "one warp, T*k <= 32"),
    (4, 256, 8, "normal", "one warp, T*k <= 32"),
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
