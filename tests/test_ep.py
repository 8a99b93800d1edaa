"""Expert parallelism, host side: the expert partition, the rank holder's
checks, the entry point's argument checks, and the decomposition itself on
two CPU ranks over gloo -- each rank's share computed by the oracle, the
shares summed by ``ep.allreduce_partial``, the sum against the whole layer.
(The shares on the GPU are checked in ``tests/test_gpu_ep.py``.)"""
import ctypes
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("E", [16, 17, 256])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_expert_ranges_partition_the_experts(E, world):
    from int4_routed_expert_renorm_b200 import ep
    ranges = [ep.expert_range(E, r, world) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == E
    assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
    sizes = [e - b for b, e in ranges]
    assert min(sizes) >= 1 and max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        ep.expert_range(E, world, world)


def test_rank_holder_checks_its_tensors():
    from int4_routed_expert_renorm_b200 import dims_for, ep
    H, I, E, S = 256, 256, 8, 1
    d = dims_for(H, I, E, 2, S)
    full = {"gate_q": torch.zeros(E + S, I, H // 2, dtype=torch.uint8), "up_q": torch.zeros(E + S, I, H // 2, dtype=torch.uint8),
            "down_q": torch.zeros(E + S, H, I // 2, dtype=torch.uint8), "gate_s": torch.zeros(E + S, I, H // 32, dtype=torch.int16),
            "up_s": torch.zeros(E + S, I, H // 32, dtype=torch.int16), "down_s": torch.zeros(E + S, H, I // 32, dtype=torch.int16)}
    for t in full.values():
        t.copy_(torch.arange(t.numel()).reshape(t.shape).to(t.dtype))
    loc = ep.local_tensors(full, d, 2, 5, True)
    assert loc["gate_q"].shape[0] == 4 and torch.equal(loc["gate_q"][:3], full["gate_q"][2:5])
    assert torch.equal(loc["down_s"][3], full["down_s"][E])
    ep.ExpertParallelLayer(d, loc, 2, 5, True)
    with pytest.raises(ValueError, match="gate_q"):
        ep.ExpertParallelLayer(d, loc, 2, 5, False)        # holds one expert too many
    with pytest.raises(ValueError):
        ep.ExpertParallelLayer(d, ep.local_tensors(full, d, 0, 3, False), 3, 3, False)


def test_layer_ep_argument_checks():
    import int4_routed_expert_renorm_b200 as m
    lib = m._lib._lib
    d = m.coli_moe_dims(6144, 2048, 256, 8, 1, 32, 4)
    f = ctypes.c_void_p(0x10000)
    w = m.coli_moe_weights(f, f, f, f, f, f, f, None)
    ws, part, x = ctypes.c_void_p(0x400000), ctypes.c_void_p(0x300000), ctypes.c_void_p(0x200000)
    n = m.coli_moe_workspace_bytes(d, 8)
    L = lambda b, e, T, p=part, flags=0: lib.coli_moe_layer_ep(ctypes.byref(d), ctypes.byref(w), b, e, 1, x, T, None,  # noqa: E731
                                                           None, flags, p, None, None, None, ws, n, None)
    assert L(0, 0, 1) == m._lib.COLI_ERR_INVALID_ARG          # empty range
    assert L(-1, 8, 1) == m._lib.COLI_ERR_INVALID_ARG
    assert L(0, 257, 1) == m._lib.COLI_ERR_INVALID_ARG
    assert L(0, 128, 1, p=None) == m._lib.COLI_ERR_INVALID_ARG
    assert L(0, 128, 1, p=ctypes.c_void_p(0x300008)) == m._lib.COLI_ERR_INVALID_ARG   # partial not 16-byte aligned
    assert L(0, 128, 9) in (m._lib.COLI_OK, m._lib.COLI_ERR_CUDA)   # the two-phase form, T <= 128
    assert L(0, 128, 129) == m._lib.COLI_ERR_UNSUPPORTED      # route + union + plan in one kernel only
    assert L(0, 128, 4, flags=0x20) in (m._lib.COLI_OK, m._lib.COLI_ERR_CUDA)   # the prefill form
    assert L(0, 128, 4, flags=0x2) == m._lib.COLI_ERR_UNSUPPORTED   # host-memory input
    assert L(0, 128, 0) == m._lib.COLI_OK                    # T = 0
    # past the checks a machine without a GPU stops at the device query
    assert L(0, 128, 4) in (m._lib.COLI_OK, m._lib.COLI_ERR_CUDA)
    assert lib.coli_moe_partial_to_bf16(part, x, 6, None) == m._lib.COLI_ERR_INVALID_ARG   # n % 4 != 0
    assert lib.coli_moe_partial_to_bf16(part, x, 0, None) == m._lib.COLI_OK


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import oracle
    import synth
    from int4_routed_expert_renorm_b200 import ep
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        shape = synth.LayerShape("small", 256, 256, 16, 4, 1, 3)
        li = synth.LayerInputs(shape, 21)
        W = oracle.ExpertWeights.from_synth(li)
        x = synth.normal_bf16(21, 5, synth.X_IN, (3, 256))
        res = synth.normal_bf16(21, 6, synth.X_IN, (3, 256))
        lay = oracle.moe_layer(W, x, shape.n_experts, shape.top_k, shape.n_shared, router_w=li.router_w())
        ids, w = lay["ids"], lay["w"]
        b, e = ep.expert_range(shape.n_experts, rank, world)
        # this rank's share: its routed experts' weighted outputs (+ the shared
        # experts and the residual on rank 0), float64 as the oracle sums
        wl = np.where((ids >= b) & (ids < e), w, 0.0)
        _, part = oracle.moe_ffn_combine(W, x, ids, wl, shape.n_experts, shape.n_shared if rank == 0 else 0,
                                         res if rank == 0 else None, return_f64=True)
        t = torch.from_numpy(part.copy())
        ep.allreduce_partial(t)
        _, whole = oracle.moe_ffn_combine(W, x, ids, w, shape.n_experts, shape.n_shared, res, return_f64=True)
        q.put((rank, t.numpy().copy(), whole))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_expert_parallel_shares_sum_to_the_layer_over_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    whole = got[0][2]
    for rank, summed, _ in got:
        # the float64 shares summed in another order: equal to rounding
        assert np.abs(summed - whole).max() <= 1e-12 * np.abs(whole).max(), rank
