"""The multi-GPU path of bench.py is replicas (the MoE step has no exchange):
every rank runs its own batches on its own copy of the layer, and the job's
throughput is all ranks' tokens over the slowest rank's device time.  These
tests run that host logic on two CPU processes over gloo."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import bench
    import synth
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        batches = bench.rank_batches(rank, 4)
        x = synth.activations(synth.TINY, 0, batches[0])
        local_ms = 10.0 + 5.0 * rank
        slowest = bench.max_over_ranks(local_ms, world, "cpu")
        value = bench.job_throughput(world, synth.TINY.tokens, 7, slowest)
        q.put((rank, batches, x.tobytes(), slowest, value))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_replicas_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(2):
        rank, batches, xb, slowest, value = q.get(timeout=120)
        out[rank] = (batches, xb, slowest, value)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # disjoint batches, hence different inputs on the two ranks
    assert set(out[0][0]).isdisjoint(out[1][0])
    assert out[0][1] != out[1][1]
    # both ranks agree on the slowest rank's time and on the job throughput
    assert out[0][2] == out[1][2] == 15.0
    expect = 2 * 4 * 7 / (15.0 / 1e3)
    assert out[0][3] == pytest.approx(expect) and out[1][3] == pytest.approx(expect)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")

    class A:
        workload = "tiny_h256_i128_e16_k2_t4"
        cpu_seconds = 0.1
        gpus = 2
        steps = 1
        warmup = 3
    assert bench.run_reference(A()) == 0
    assert capsys.readouterr().out == ""


def test_single_rank_helpers_need_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
    assert bench.rank_batches(0, 3) == [0, 1, 2] and bench.rank_batches(2, 3) == [6, 7, 8]
    assert bench.job_throughput(1, 4, 10, 20.0) == pytest.approx(2000.0)
    assert np.isfinite(bench.job_throughput(8, 1, 1, 0.5))
