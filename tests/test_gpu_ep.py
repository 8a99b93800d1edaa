"""Expert parallelism on the GPU (split-K form up to 8 tokens, two-phase form
up to 128, the prefill form at any size), with the ranks emulated one after another
on one device (each rank's call is independent: nothing waits on another
rank).  Each rank holds a contiguous range of the routed experts (rank 0 also
the shared ones and the residual) and computes its fp32 share with
coli_moe_layer_ep; the shares are summed in rank order and rounded once with
coli_moe_partial_to_bf16.  Checks: every rank routes exactly as the whole
layer does (logits, ids, weights bit-exact), the summed output against the
oracle within the layer tolerance and against the whole layer's output, and
the rounding kernel bit-exact against round-to-nearest-even."""
import numpy as np
import pytest
import torch

import oracle
import synth
import synth.gpu as sg
from tests._gpu import OUT_REL_TOL, bits, needs_gpu, oracle_weights, to_dev_bits
from tests.test_gpu_parity import _small_shape, lib  # noqa: F401

pytestmark = [pytest.mark.gpu, needs_gpu]

PRENORM = 0x1


def _ep_run(lib, shape, full, li, x_bits, world, res_bits=None, flags=0, seed=0):
    from int4_routed_expert_renorm_b200 import ep
    d = lib.dims_for(shape.hidden, shape.inter, shape.n_experts, shape.top_k, shape.n_shared, shape.group, shape.bits)
    T, H, E, k = shape.tokens, shape.hidden, shape.n_experts, shape.top_k
    rw = torch.from_numpy(li.router_w()).cuda()
    b = li.bias()
    bias = None if b is None else torch.from_numpy(b).cuda()
    x = to_dev_bits(x_bits)
    res = None if res_bits is None else to_dev_bits(res_bits)
    total = torch.zeros((T, H), dtype=torch.float32, device="cuda")
    routing = []
    for r in range(world):
        lo, hi = ep.expert_range(E, r, world)
        layer = ep.ExpertParallelLayer(d, ep.local_tensors(full, d, lo, hi, r == 0), lo, hi, r == 0, rw, bias)
        part = torch.empty((T, H), dtype=torch.float32, device="cuda")
        lg = torch.empty((T, E), dtype=torch.float32, device="cuda")
        ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
        w = torch.empty((T, k), dtype=torch.float32, device="cuda")
        layer.partial(x, part, layer.workspace(T), residual=res, flags=flags, logits_out=lg, topk_ids_out=ids,
                      topk_w_out=w)
        st, fl = lib.coli_moe_get_status()
        assert st == 0 and fl == 0
        total += part
        routing.append((lg.cpu().numpy(), ids.cpu().numpy(), w.cpu().numpy()))
        del layer
    out = torch.empty((T, H), dtype=torch.int16, device="cuda")
    lib.coli_moe_partial_to_bf16(total, out)
    return bits(out), total.cpu().numpy(), routing


def _whole(lib, shape, full, li, x_bits, res_bits=None, flags=0):
    d = lib.dims_for(shape.hidden, shape.inter, shape.n_experts, shape.top_k, shape.n_shared, shape.group, shape.bits)
    b = li.bias()
    layer = lib.MoELayer(d, full, torch.from_numpy(li.router_w()).cuda(), None if b is None else torch.from_numpy(b).cuda())
    T = shape.tokens
    x = to_dev_bits(x_bits)
    out = torch.empty_like(x)
    lg = torch.empty((T, shape.n_experts), dtype=torch.float32, device="cuda")
    ids = torch.empty((T, shape.top_k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, shape.top_k), dtype=torch.float32, device="cuda")
    layer.forward(x, out, layer.workspace(T), residual=None if res_bits is None else to_dev_bits(res_bits),
                  flags=flags, logits_out=lg, topk_ids_out=ids, topk_w_out=w)
    return bits(out), (lg.cpu().numpy(), ids.cpu().numpy(), w.cpu().numpy())


def _rel(a_bits, b_bits):
    a, b = oracle.bf16_bits_to_f64(a_bits), oracle.bf16_bits_to_f64(b_bits)
    return np.abs(a - b).max() / np.abs(b).max()


PREFILL = 0x20


@pytest.mark.parametrize("T,world,flags", [(1, 2, 0), (5, 3, 0), (8, 2, PRENORM), (3, 4, PRENORM),
                                           (20, 3, 0), (64, 2, PRENORM), (100, 4, 0),
                                           (40, 2, PREFILL), (300, 3, PREFILL | PRENORM), (200, 4, PREFILL)])
def test_expert_parallel_small(lib, T, world, flags):
    shape = _small_shape(tokens=T, hidden=512, inter=256, n_experts=16, top_k=4, n_shared=1)
    full = sg.expert_tensors(shape, 23)
    li = synth.LayerInputs(shape, 23)
    x = synth.normal_bf16(23, 5, synth.X_IN, (T, 512))
    res = synth.normal_bf16(23, 6, synth.X_IN, (T, 512))
    out, total, routing = _ep_run(lib, shape, full, li, x, world, res, flags)
    ref_out, ref_routing = _whole(lib, shape, full, li, x, res, flags)
    for lg, ids, w in routing:
        assert np.array_equal(lg, ref_routing[0]) and np.array_equal(ids, ref_routing[1])
        assert np.array_equal(w, ref_routing[2])
    W = oracle_weights(shape, seed=23)
    xin = oracle.rms_norm(x) if flags & PRENORM else x
    ref = oracle.moe_ffn_combine(W, xin, ref_routing[1], ref_routing[2], shape.n_experts, shape.n_shared, res)
    err, err_whole = _rel(out, ref), _rel(out, ref_out)
    print(f"expert-parallel T={T} over {world} ranks: vs oracle {err:.3e}, vs the whole layer {err_whole:.3e}")
    assert err <= OUT_REL_TOL and err_whole <= OUT_REL_TOL
    # the rounding kernel: round-to-nearest-even of the fp32 sum, bit for bit
    assert np.array_equal(out, oracle.f64_to_bf16_bits(total.astype(np.float64)))


@pytest.mark.parametrize("T,world,form", [(1, 2, 0), (4, 4, 0), (24, 2, 0), (160, 2, PREFILL)])
def test_expert_parallel_glm_shape(lib, T, world, form):
    """The GLM-5.2-shaped layer (H 6144, I 2048, top-8, one shared expert) with
    16 routed experts resident, spread over 2 and 4 ranks (24 tokens: the
    two-phase form; 160 tokens forced into the prefill form)."""
    base = synth.DECODE_B1_E16
    shape = synth.LayerShape(base.name, base.hidden, base.inter, base.n_experts, base.top_k, base.n_shared, T)
    full = sg.expert_tensors(shape, 0)
    li = synth.LayerInputs(shape, 0)
    x = np.concatenate([synth.activations(shape, 0, b)[:1] for b in range(T)])
    out, _, routing = _ep_run(lib, shape, full, li, x, world, x, PRENORM | form)
    ref_out, ref_routing = _whole(lib, shape, full, li, x, x, PRENORM | form)
    for lg, ids, w in routing:
        assert np.array_equal(ids, ref_routing[1]) and np.array_equal(w, ref_routing[2])
    err = _rel(out, ref_out)
    print(f"expert-parallel GLM shape T={T} over {world} ranks: vs the whole layer {err:.3e}")
    assert err <= OUT_REL_TOL
    del full
    torch.cuda.empty_cache()


@pytest.mark.parametrize("kw", [dict(tokens=4, group=64), dict(tokens=40, group=64), dict(tokens=6, bits=8)],
                         ids=["gs64-splitk", "gs64-two-phase", "int8"])
def test_expert_parallel_containers(lib, kw):
    """The gs64 and int8 containers through the expert-parallel share."""
    shape = _small_shape(hidden=512, inter=512, n_experts=12, top_k=3, n_shared=1, **kw)
    T = shape.tokens
    full = sg.expert_tensors(shape, 24)
    li = synth.LayerInputs(shape, 24)
    x = synth.normal_bf16(24, 5, synth.X_IN, (T, 512))
    out, _, routing = _ep_run(lib, shape, full, li, x, 3, x)
    ref_out, ref_routing = _whole(lib, shape, full, li, x, x)
    for lg, ids, w in routing:
        assert np.array_equal(ids, ref_routing[1]) and np.array_equal(w, ref_routing[2])
    W = oracle_weights(shape, seed=24)
    ref = oracle.moe_ffn_combine(W, x, ref_routing[1], ref_routing[2], shape.n_experts, shape.n_shared, x)
    err = _rel(out, ref)
    print(f"expert-parallel {kw}: vs oracle {err:.3e}, vs the whole layer {_rel(out, ref_out):.3e}")
    assert err <= OUT_REL_TOL and _rel(out, ref_out) <= OUT_REL_TOL
