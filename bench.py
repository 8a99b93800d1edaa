#!/usr/bin/env python
"""Throughput of the routed-expert MoE layer (Route -> Union -> int4 SwiGLU FFN -> combine) on B200.

    python bench.py [--gpus N --steps K --warmup W] [--workload NAME] [--impl colimoe|reference]

One step = one pass of the whole layer (pre-norm/logits, route, union, expert
FFN, combine) over one batch of seeded synthetic input already resident in
HBM; for the 16-layer stack a step is one forward through all 16 layers.
Inputs rotate over 8 batches and L2 is flushed before every step, outside
the timed events: a 256 MiB write, then a 256 MiB read, so the step starts
with clean unrelated lines in L2 (no hits, and no write-back of the flush's
dirty lines inside the timed region).  Each step is timed with CUDA events on the
launching stream; the total is the sum over K steps, max over ranks.  With
N > 1 (torchrun) every rank runs its own batches on its own replica of the
layer (the path has no exchange step): value = tokens of all ranks / time.

Rank 0 prints one JSON line.  ``--impl reference`` times the CPU oracle on
the host cores instead (rank 0 only) and prints the same line with
"impl": "reference".
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "routed-MoE layer tokens/s at 1 B200; int4 weight GB/s vs HBM peak (decode)"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = synth.DECODE_B1.name
FLUSH_BYTES = 256 << 20   # > 126 MB of L2


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["colimoe", "reference"], default="colimoe")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--batches", type=int, default=8)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tier", type=int, default=0,
                    help="run a one-layer decode workload through a host-RAM expert tier with this many device "
                         "slots (the routed experts in page-locked host memory)")
    ap.add_argument("--form", choices=["auto", "decode", "prefill"], default="auto",
                    help="FFN form (COLI_PATH_*); auto lets the library choose")
    ap.add_argument("--graph", choices=["on", "off"], default="on",
                    help="replay each step from a CUDA graph captured once per input batch (the stage breakdown "
                         "then comes from separate eager steps)")
    ap.add_argument("--cpu-seconds", type=float, default=20.0, help="target length of the oracle sample")
    a = ap.parse_args()
    if a.steps is None:
        a.steps = {"glm52_layer_decode_b1": 2000, "glm52_layer_decode_b64_zipf": 400,
                   "glm52_layer_prefill_4096": 40, "glm52_stack16_decode_b4": 200,
                   "glm52_layer_prefill_512_e32": 50, "glm52_layer_decode_b1_gs64": 2000,
                   "glm52_layer_prefill_4096_gs64": 40,
                   "glm52_layer_int8_decode_b1": 1000, "glm52_layer_prefill_4096_router": 40}.get(a.workload, 20)
    a.warmup = max(a.warmup, 3)
    return a


# DRAM bytes (read + write) per launch of the dominant kernel, from one ncu
# capture, with a digest of the kernel sources that capture ran on:
# (workload, FFN form) -> (bytes, digest).  While the sources differ from that
# digest (a kernel changed since the counters were taken) the line reports
# null.  The batch-1 capture ran on the 16-expert variant of the layer, which
# moves the same 9 experts per step; the prefill capture on the 32-expert,
# 512-token variant (same tile shapes), where DRAM traffic was 1.067x the
# algorithmic bytes of the gate/up launch; the 4096-token figure is that ratio
# times its own algorithmic bytes (257 experts' gate+up codes and scales,
# 36,864 gathered rows, h written).
_SK_SOURCES = "1b3dc4bd04b4489a"
_PF_SOURCES = "70d5aa5efa5b0120"
_PF_RATIO = (532.818432e6 + 18.652416e6) / (33 * 2 * 6684672 + 4608 * 6144 * 2 + 4608 * 2048 * 2)
_PF_4096 = _PF_RATIO * (257 * 2 * 6684672 + 36864 * 6144 * 2 + 36864 * 2048 * 2)
TRAFFIC = {("glm52_layer_decode_b1", "decode"): (191.196416e6 + 5.173248e6, _SK_SOURCES),
           ("glm52_layer_decode_b1_e16", "decode"): (191.196416e6 + 5.173248e6, _SK_SOURCES),
           ("glm52_layer_prefill_512_e32", "prefill"): (532.818432e6 + 18.652416e6, _PF_SOURCES),
           # the two-phase decode kernel (the same sources as the split-K one)
           ("glm52_layer_decode_b64_zipf_e32", "decode"): (758.119168e6 + 16.141824e6, _SK_SOURCES),
           ("glm52_layer_prefill_4096", "prefill"): (_PF_4096, _PF_SOURCES),
           # same gate/up launch: all 256 routed experts and the shared one touched, 36,864 rows
           ("glm52_layer_prefill_4096_router", "prefill"): (_PF_4096, _PF_SOURCES)}
# the sources each captured kernel is built from
_KERNEL_FILES = {"decode": ("common.cuh", "k_ffn_decode.cuh", "k_ffn_splitk.cuh"),
                 "prefill": ("common.cuh", "k_ffn_decode.cuh", "k_ffn_prefill.cuh")}


def kernel_sources_digest(files=None) -> str:
    """First 16 hex digits of the sha256 over the named kernel sources (all of
    them by default): file name, then contents, in name order."""
    import glob
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "int4_routed_expert_renorm_b200", "csrc")
    paths = sorted(glob.glob(os.path.join(csrc, "*"))) if files is None else sorted(
        os.path.join(csrc, f) for f in files)
    for f in paths:
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_for(workload: str, form: str):
    """The captured DRAM bytes per launch, or None when there is no capture of
    the current sources of that kernel."""
    entry = TRAFFIC.get((workload, form))
    if entry is None or kernel_sources_digest(_KERNEL_FILES[form]) != entry[1]:
        return None
    return entry[0]


def splitk_form(shape) -> bool:
    """The library's decode form for batches of <= 8 tokens (I a multiple of 256)."""
    return shape.tokens <= 8 and shape.inter % 256 == 0


def prefill_form(shape) -> bool:
    """The library takes the prefill (tcgen05) form once a batch averages >= 32
    tokens per expert; the prefill workloads are the ones that do."""
    P = shape.tokens * shape.top_k
    return shape.tokens >= 32 and P >= 32 * min(shape.n_experts, P)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d["bf16_tflops_sustained"], "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.proc, self.path, self.index = None, None, index
        try:
            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(index), "-lms", "100"], stdout=open(self.path, "w"),
                                         stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self, t0: float, t1: float):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for ln in open(self.path):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = time.mktime(time.strptime(f[0].split(".")[0], "%Y/%m/%d %H:%M:%S")) + float("0." + f[0].split(".")[1])
                rows.append((ts, float(f[2]), float(f[3]), f[6:10], f[5]))
            except (ValueError, IndexError):
                continue
        os.unlink(self.path)
        inside = [r for r in rows if t0 - 0.15 <= r[0] <= t1 + 0.15]
        use = inside if inside else rows
        if not use:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in use for i, v in enumerate(r[3]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[1] for r in use), "sm_max_mhz": max(r[2] for r in use),
                "reasons": reasons, "samples": len(use), "samples_in_window": len(inside)}


# ------------------------------------------------------------------ the oracle leg (CPU)

_KINDS = {"gate": (synth.GATE_Q, synth.GATE_S), "up": (synth.UP_Q, synth.UP_S), "down": (synth.DOWN_Q, synth.DOWN_S)}


def _oracle_tokens(name: str, batch: int, toks: list[int], warm: int = 0) -> tuple[float, int]:
    """Time the plain-C oracle (oracle/c/moe_ref.c, -O2, one thread) on tokens
    `toks` of input batch `batch` of a workload, one token per call, each on
    the first layer of the workload: the weights of the experts a token
    selects are generated beforehand (untimed); the timed call is the C
    oracle's whole layer (logits or given logits, route, union, expert FFN,
    combine; pre-norm for the stack).  The first `warm` calls run untimed
    (warm-up).  Returns (seconds, timed calls)."""
    import oracle.cref as cr
    cr.build()
    shape = synth.WORKLOADS[name]
    li = synth.LayerInputs(shape, 0, 0)
    rw = None if shape.logits_in else li.router_w()
    bias = li.bias()
    x = synth.activations(shape, 0, batch)
    lg = None
    if shape.logits_in:
        lg = synth.normal_f32(0, 1000 + batch, synth.LOGITS_IN, (shape.tokens, shape.n_experts), 1.0)
    elapsed = 0.0
    for n_call, t in enumerate(toks):
        xt = x[t:t + 1]
        xin = cr.rms_norm(xt) if shape.prenorm else xt
        lt = None if lg is None else lg[t:t + 1]
        l32 = lt if lt is not None else cr.router_logits(xin, rw)[1]
        ids = cr.route(l32, shape.top_k, bias)[0]
        need = sorted(set(ids.ravel().tolist()) | set(range(shape.n_experts, shape.n_total)))
        held = {(kind, e): (li.expert_codes(q, e), li.expert_scales(sc, e)) for kind, (q, sc) in _KINDS.items()
                for e in need}
        t0 = time.perf_counter()
        xin = cr.rms_norm(xt) if shape.prenorm else xt
        cr.moe_layer_experts(lambda kind, e: held[(kind, e)], shape.hidden, shape.inter, xin, shape.n_experts,
                             shape.top_k, shape.n_shared, shape.group, shape.bits, router_w=rw, bias=bias,
                             logits_in=lt, residual_bits=xt if shape.prenorm else None, experts=need)
        if n_call >= warm:
            elapsed += time.perf_counter() - t0
    return elapsed, len(toks) - min(warm, len(toks))


def cpu_model() -> str:
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_sample(shape: synth.LayerShape, seconds: float, warm: int = 0):
    """Time the CPU oracle, as it stands, on a bounded sample of the workload.

    The plain-C oracle, one token per call.  Decode and stack workloads: one
    core, tokens taken in turn from the rotating input batches until about
    `seconds` of oracle time.  Prefill workloads (thousands of tokens): one
    process per host core (spawned, so no CUDA state is inherited), each
    timing its own share of tokens; throughput = all tokens over the longest
    worker's oracle time.  The stack times one layer per token and scales by
    the layer count.  `warm` untimed warm-up calls precede the timed ones
    (in every process).  Returns (tokens/s, cores, timed calls, description)."""
    per_call = 4.0 if shape.hidden >= 4096 else 0.001      # rough C-oracle seconds per token (GLM shape)
    ncores = os.cpu_count() or 1
    parallel = shape.tokens >= 512 and ncores > 1
    if not parallel:
        n = max(1, min(64, int(seconds / per_call)))
        toks = [(i // shape.tokens, i % shape.tokens) for i in range(n)]   # (batch, token) in turn
        if shape.tokens > 1:     # spread the sample over the batch's tokens
            step = max(1, shape.tokens // max(1, n))
            toks = [(i // shape.tokens, (i * step) % shape.tokens) for i in range(n)]
        el, calls = 0.0, 0
        for i, b in enumerate(sorted({bt for bt, _ in toks})):
            tl = [t for bb, t in toks if bb == b]
            w = warm if i == 0 else 0
            e, c = _oracle_tokens(shape.name, b, tl[:1] * w + tl, w)
            el += e
            calls += c
        el *= shape.layers
        cores = 1
        desc = (f"{calls} calls of 1 token each of {shape.name} (rotating input batches); plain C oracle "
                f"(gcc -O2, -ffp-contract=off), 1 thread")
    else:
        import multiprocessing as mp
        per_worker = max(1, int(seconds / per_call))
        tok_lists = [[(w * per_worker + i) * 131 % shape.tokens for i in range(per_worker)] for w in range(ncores)]
        ctx = mp.get_context("spawn")
        with ctx.Pool(ncores) as pool:
            res = pool.starmap(_oracle_tokens, [(shape.name, 0, tl[:1] * warm + tl, warm) for tl in tok_lists])
        el = max(e for e, _ in res)
        calls = sum(c for _, c in res)
        cores = ncores
        desc = (f"{calls} calls of 1 token each of {shape.name}, {per_worker} per process on {ncores} processes "
                f"(spawned), throughput = tokens / longest process; plain C oracle (gcc -O2, -ffp-contract=off)")
    desc += (f"{'; one layer timed, x' + str(shape.layers) + ' for the stack' if shape.layers > 1 else ''}"
             f"; touched experts' weights generated untimed"
             f"{f'; {warm} untimed warm-up call(s) first' if warm else ''}; host: {ncores} cores, {cpu_model()}")
    return calls / el, cores, calls, desc


# ---- replicas over ranks (the path has no exchange step) -------------------

def rank_batches(rank: int, nb: int) -> list[int]:
    """Seed indices of the nb rotating input batches of one rank: every rank
    draws its own batches, so ranks never process the same tokens."""
    return [rank * nb + b for b in range(nb)]


def max_over_ranks(ms: float, world: int, device) -> float:
    """A rank's device-timed milliseconds -> the maximum over all ranks."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, tokens_per_step: int, steps: int, ms: float) -> float:
    """Whole-job tokens/s: the tokens of all ranks over the slowest rank's time."""
    return world * tokens_per_step * steps / (ms / 1e3)


def workload_config(shape, rotating: int) -> dict:
    """The `config` of both arms' bench lines: the workload and how it was fed."""
    return {"workload": shape.name, "tokens": shape.tokens, "hidden": shape.hidden, "inter": shape.inter,
            "experts": shape.n_experts, "top_k": shape.top_k, "shared": shape.n_shared, "layers": shape.layers,
            "group": shape.group, "code_bits": shape.bits, "rotating_batches": rotating,
            "l2": "GPU arm: L2 flushed before every step (256 MiB write, then 256 MiB read), outside the timed events"}


def run_reference(a):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    shape = synth.WORKLOADS[a.workload]
    # warm-up: up to 3 untimed oracle calls (each takes seconds at the GLM shape)
    warm = max(1, min(a.warmup, 3))
    v, cores, calls, desc = oracle_sample(shape, max(5.0, a.cpu_seconds), warm)
    # a step here is one timed oracle call (one token; for the stack, one
    # token through all layers)
    line = {"metric": METRIC, "value": v, "unit": UNIT, "n_gpus": a.gpus, "steps": calls, "warmup": warm,
            "ms_per_step": 1e3 / v, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": workload_config(shape, a.batches),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ the GPU leg

def main():
    a = parse()
    if a.impl == "reference":
        return run_reference(a)
    import torch
    import torch.distributed as dist

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))

    import int4_routed_expert_renorm_b200 as cm
    import synth.gpu as sg

    shape = synth.WORKLOADS[a.workload]
    T, H, I, E, k, S = shape.tokens, shape.hidden, shape.inter, shape.n_experts, shape.top_k, shape.n_shared
    dims = cm.dims_for(H, I, E, k, S, shape.group, shape.bits)
    layers = []
    for l in range(shape.layers):
        li = synth.LayerInputs(shape, 0, l)
        rw = None if shape.logits_in else torch.from_numpy(li.router_w()).cuda()
        b = li.bias()
        bias = None if b is None else torch.from_numpy(b).cuda()
        if a.tier:
            if shape.layers != 1:
                raise SystemExit("--tier runs one-layer workloads")
            full = sg.expert_tensors(shape, 0, l)
            layers.append(cm.tier.TieredLayer(dims, full, a.tier, rw, bias))
            del full
            torch.cuda.empty_cache()
        else:
            layers.append(cm.MoELayer(dims, sg.expert_tensors(shape, 0, l), rw, bias))
    NB = a.batches
    xs = [torch.from_numpy(synth.activations(shape, 0, bi).view(np.int16)).cuda() for bi in rank_batches(rank, NB)]
    lgs = [None] * NB
    if shape.logits_in:
        lgs = [torch.from_numpy(synth.normal_f32(0, 1000 + bi, synth.LOGITS_IN, (T, E), 1.0)).cuda()
               for bi in rank_batches(rank, NB)]
    ws = layers[0].workspace(T)
    outs = [torch.empty((T, H), dtype=torch.int16, device="cuda") for _ in range(2)]
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    flush_rd = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    flush_sink = torch.empty(1, dtype=torch.float32, device="cuda")

    def flush_l2():
        # write a buffer larger than L2, then read another one: L2 ends up
        # holding clean, unrelated lines, so the timed step neither hits in L2
        # nor pays for writing back the flush's dirty lines
        flush.zero_()
        torch.sum(flush_rd, dim=0, out=flush_sink)
    flags = cm._lib.COLI_LAYER_PRENORM if shape.prenorm else 0
    flags |= {"auto": 0, "decode": cm._lib.COLI_PATH_DECODE, "prefill": cm._lib.COLI_PATH_PREFILL}[a.form]

    def step(bi, x=None, out=None, host=False):
        # host: x (and the first layer's residual) and out are page-locked host
        # buffers, read and written by the library's own kernels
        x = xs[bi] if x is None else x
        hx = cm._lib.COLI_LAYER_HOST_X if host else 0
        ho = cm._lib.COLI_LAYER_HOST_OUT if host else 0
        if shape.layers == 1:
            o = outs[0] if out is None else out
            layers[0].forward(x, o, ws, logits_in=lgs[bi], flags=flags | hx | ho)
            return o
        h = x
        for li_, lay in enumerate(layers):
            last = li_ == len(layers) - 1
            o = outs[li_ % 2] if (out is None or not last) else out
            f = flags | (hx if li_ == 0 else 0) | (ho if last else 0)
            lay.forward(h, o, ws, residual=h if shape.prenorm else None, flags=f)
            h = o
        return h

    # union size per batch (first layer), for the bytes-touched accounting
    U = []
    ids_buf = torch.empty((T, k), dtype=torch.int32, device="cuda")
    for bi in range(NB):
        layers[0].forward(xs[bi], outs[0], ws, logits_in=lgs[bi], flags=flags, topk_ids_out=ids_buf)
        U.append(int(torch.unique(ids_buf).numel()))
    st, fl = cm.coli_moe_get_status()
    if fl:
        raise RuntimeError(f"device status flags {fl:#x} after the first pass")
    u_stack = []
    if shape.layers > 1:  # union size of every layer, batch 0 (one untimed forward)
        h = xs[0]
        for li_, lay in enumerate(layers):
            o = outs[li_ % 2]
            lay.forward(h, o, ws, residual=h, flags=flags, topk_ids_out=ids_buf)
            u_stack.append(int(torch.unique(ids_buf).numel()))
            h = o

    for i in range(a.warmup):
        step(i % NB)
    torch.cuda.synchronize()

    K = a.steps
    M = min(K, 64)
    use_graph = a.graph == "on"
    graphs = []
    launches_per_step = None
    stage = [[torch.cuda.Event(enable_timing=True) for _ in range(9)] for _ in range(M)]
    for evs in stage:  # create the events (they exist once recorded)
        for e in evs:
            e.record()
    torch.cuda.synchronize()
    if use_graph:
        # stage breakdown from eager steps (events cannot sit inside the graphs)
        for i in range(M):
            flush_l2()
            cm.coli_moe_set_stage_events(stage[i])
            step(i % NB)
        torch.cuda.synchronize()
        cm.coli_moe_launch_count(reset=True)
        for bi in range(NB):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step(bi)
            graphs.append(g)
        launches_per_step = cm.coli_moe_launch_count(reset=True) // NB
        for bi in range(NB):   # warm replays
            graphs[bi].replay()
        torch.cuda.synchronize()

    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local) if rank == 0 else None
    time.sleep(0.3 if sampler else 0)
    tier0 = layers[0].state_arrays() if a.tier else None
    cm.coli_moe_launch_count(reset=True)
    t_wall0 = time.time()
    for i in range(K):
        flush_l2()
        ev_s[i].record()
        if use_graph:
            graphs[i % NB].replay()
        else:
            if i < M:
                cm.coli_moe_set_stage_events(stage[i])
            step(i % NB)
        ev_e[i].record()
    torch.cuda.synchronize()
    t_wall1 = time.time()
    launches = launches_per_step * K if use_graph else cm.coli_moe_launch_count()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop(t_wall0, t_wall1) if sampler else None
    st, fl = cm.coli_moe_get_status()
    if fl:
        raise RuntimeError(f"device status flags {fl:#x} in the timed region")

    step_ms = [ev_s[i].elapsed_time(ev_e[i]) for i in range(K)]
    total_ms = max_over_ranks(sum(step_ms), world, "cuda")
    value = job_throughput(world, T, K, total_ms)
    tier = None
    if a.tier:
        # the timed steps' placement: hits, misses, and the expert bytes the
        # misses copied over the host link
        t1 = layers[0].state_arrays()
        hits, misses = t1["hits"] - tier0["hits"], t1["misses"] - tier0["misses"]
        fill_b = (t1["fills"] - tier0["fills"]) * shape.expert_bytes() / K
        tier = {"slots": a.tier, "experts": E, "hit_rate": hits / max(1, hits + misses), "hits_per_step": hits / K,
                "misses_per_step": misses / K, "fill_bytes_per_step": fill_b,
                "fill_gbs_over_the_step": fill_b / (total_ms / K / 1e3) / 1e9}

    # dominant kernel, timed live on the launching stream (stage 5 -> 6): the
    # decode form's one persistent FFN launch (gate/up, down and, for T <= 4,
    # the combine), or the prefill form's gate/up GEMM
    gu_ms = [stage[i][5].elapsed_time(stage[i][6]) for i in range(M)]
    gu_avg = statistics.mean(gu_ms)
    stage_names = ["prep", "logits", "route", "union", "plan", "gate_up", "down", "combine"]
    stage_ms = {n: statistics.mean(stage[i][j].elapsed_time(stage[i][j + 1]) for i in range(M))
                for j, n in enumerate(stage_names)}
    hbm, tf_burst, tf_sus, src = peaks()
    P = T * k
    u_step = [U[i % NB] for i in range(M)]  # the first layer of each step carries the stage events
    form = a.form if a.form != "auto" else ("prefill" if prefill_form(shape) else "decode")
    per_mat = H * I // 2 + (H * I // shape.group) * 2   # codes + scales of one matrix
    if form == "prefill" and not prefill_form(shape):
        # prefill form on a decode-sized batch: the gate/up GEMM streams the
        # gate and up matrices of every touched expert
        rows = P + S * T
        per_launch = [(u + S) * 2 * per_mat + (P + T) * H * 2 + rows * I * 2 for u in u_step]
        achieved = statistics.mean(b / (ms / 1e3) / 1e9 for b, ms in zip(per_launch, gu_ms))
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                "traffic": None,
                "kernel": "ffn_prefill_kernel<2> (gate/up grouped GEMM, tcgen05 kind::f16, A in TMEM)",
                "algorithmic": "gate and up codes + fp16 scales of every unique and shared expert "
                               "+ gathered x read + h write",
                "peak_kind": f"{src} HBM copy"}
    elif form == "prefill":
        flops = 2 * 2 * H * I * (P + S * T)
        achieved = flops / (gu_avg / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": tf_burst, "unit": "TFLOP/s",
                "frac": achieved / tf_burst, "frac_of_sustained": achieved / tf_sus, "traffic": None,
                "kernel": "ffn_prefill_kernel<2> (gate/up grouped GEMM, tcgen05 kind::f16, A in TMEM)",
                "algorithmic": f"{flops} FLOP per launch = 4*H*I per (pair or shared row)",
                "peak_kind": f"{src} burst bf16"}
    elif splitk_form(shape):
        act = T * H * 2 * (3 if shape.prenorm else 2)      # x read, out write (+ residual read)
        per_launch = [(u + S) * shape.expert_bytes() + act for u in u_step]
        achieved = statistics.mean(b / (ms / 1e3) / 1e9 for b, ms in zip(per_launch, gu_ms))
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                "traffic": None,
                "kernel": "ffn_splitk_kernel (decode form for T <= 8: gate/up, split-K down and combine in one "
                          "launch)",
                "algorithmic": "int4 codes + fp16 scales of every unique and shared expert (3 matrices) "
                               "+ x read + out write" + (" + residual read" if shape.prenorm else ""),
                "peak_kind": f"{src} HBM copy"}
    else:
        rows = P + S * T
        fused_combine = T <= 4
        per_launch = [(u + S) * shape.expert_bytes() + T * H * 2 + rows * (2 * I * 2 + H * 4)
                      + (rows * H * 4 + T * H * 2 if fused_combine else 0) for u in u_step]
        achieved = statistics.mean(b / (ms / 1e3) / 1e9 for b, ms in zip(per_launch, gu_ms))
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                "traffic": None,
                "kernel": "ffn_fused_kernel (decode form: gate/up, down" + (", combine" if fused_combine else "")
                          + " in one launch)",
                "algorithmic": "int4 codes + fp16 scales of every unique and shared expert (3 matrices) "
                               "+ x read + h write/read + y write" + (" + y read + out write" if fused_combine else ""),
                "peak_kind": f"{src} HBM copy"}

    roof["traffic"] = traffic_for(shape.name, form)
    # the same figure against the nominal spec (8 TB/s HBM3e; 2.25 PFLOP/s dense bf16), for context
    spec = 8000.0 if roof["unit"] == "GB/s" else 2250.0
    roof["frac_of_spec"] = roof["achieved"] / spec
    roof["spec"] = spec

    # int4 bytes touched per step (all three matrices of every unique + shared expert)
    exp_bytes = shape.expert_bytes()
    if shape.layers == 1:
        bytes_step = statistics.mean((U[i % NB] + S) * exp_bytes for i in range(K))
    else:
        bytes_step = sum((u + S) * exp_bytes for u in u_stack)
    int4_gbs = bytes_step / (statistics.mean(step_ms) / 1e3) / 1e9

    # end to end through the public API with host buffers
    xh = [torch.empty((T, H), dtype=torch.int16, pin_memory=True) for _ in range(NB)]
    for bi in range(NB):
        xh[bi].copy_(xs[bi].cpu())
    lh = [None] * NB
    if shape.logits_in:
        lh = [lgs[bi].cpu().pin_memory() for bi in range(NB)]
    oh = torch.empty((T, H), dtype=torch.int16, pin_memory=True)
    xd = torch.empty((T, H), dtype=torch.int16, device="cuda")
    ld = torch.empty((T, E), dtype=torch.float32, device="cuda") if shape.logits_in else None
    od = torch.empty((T, H), dtype=torch.int16, device="cuda")
    K2 = min(K, 500)
    e2e_ms = []
    es = [torch.cuda.Event(enable_timing=True) for _ in range(K2)]
    ee = [torch.cuda.Event(enable_timing=True) for _ in range(K2)]

    def e2e_step(bi):
        if ld is not None:
            lgs_save = lgs[bi]
            lgs[bi] = ld
        step(bi, x=xd, out=od)
        if ld is not None:
            lgs[bi] = lgs_save

    g_e2e = None
    if use_graph:   # one graph on the static device buffers the host copies fill
        e2e_step(0)
        torch.cuda.synchronize()
        g_e2e = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_e2e):
            e2e_step(0)
    def e2e_run(graph):
        for i in range(K2):
            bi = i % NB
            flush_l2()
            es[i].record()
            xd.copy_(xh[bi], non_blocking=True)
            if ld is not None:
                ld.copy_(lh[bi], non_blocking=True)
            if graph is not None:
                graph.replay()
            else:
                e2e_step(bi)
            oh.copy_(od, non_blocking=True)
            ee[i].record()
        torch.cuda.synchronize()
        ms = max_over_ranks(sum(es[i].elapsed_time(ee[i]) for i in range(K2)), world, "cuda")
        return job_throughput(world, T, K2, ms)

    io = {"h2d_bytes_per_step": T * H * 2 + (T * E * 4 if shape.logits_in else 0), "d2h_bytes_per_step": T * H * 2}
    e2e_copies = {"value": e2e_run(g_e2e), "unit": UNIT, **io,
                  "how": ("cudaMemcpyAsync of x in and out back around a CUDA graph of the layer call(s)"
                          if g_e2e is not None else "cudaMemcpyAsync around eager calls")}

    # the same with the input and the output in page-locked host memory, read
    # and written by the library's kernels (COLI_LAYER_HOST_X | _HOST_OUT):
    # the transfers are inside the layer call, no copy engine involved
    def e2e_host_step(bi):
        if ld is not None:
            lgs_save = lgs[bi]
            lgs[bi] = ld
        step(bi, x=xh[bi], out=oh, host=True)
        if ld is not None:
            lgs[bi] = lgs_save

    g_host = None
    if use_graph:   # one graph per rotating batch: each reads its own host rows
        for bi in range(NB):
            e2e_host_step(bi)
        torch.cuda.synchronize()
        g_host = []
        for bi in range(NB):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                e2e_host_step(bi)
            g_host.append(g)

    def e2e_host_run(graphs):
        for i in range(K2):
            bi = i % NB
            flush_l2()
            es[i].record()
            if ld is not None:
                ld.copy_(lh[bi], non_blocking=True)
            if graphs is not None:
                graphs[bi].replay()
            else:
                e2e_host_step(bi)
            ee[i].record()
        torch.cuda.synchronize()
        ms = max_over_ranks(sum(es[i].elapsed_time(ee[i]) for i in range(K2)), world, "cuda")
        return job_throughput(world, T, K2, ms)

    e2e = {"value": e2e_host_run(g_host), "unit": UNIT, **io,
           "how": ("CUDA graph of the layer call(s) with x read from and out written to page-locked host memory "
                   "by the library's kernels" if g_host is not None else "eager calls, host-memory x and out")}
    # the same through eager calls: the host side of every call (argument
    # checks, tensor-map encoding, launches) inside the timed region
    e2e_eager = ({"value": e2e_host_run(None), "unit": UNIT, **io, "how": "eager calls, host-memory x and out"}
                 if g_host is not None else None)

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        v, cores, calls, desc = oracle_sample(shape, a.cpu_seconds)
        cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": a.warmup,
            "ms_per_step": total_ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic", "ffn_form": form, "cuda_graph": use_graph,
            "config": dict(workload_config(shape, NB), **({"tier_slots": a.tier} if a.tier else {})),
            "union_per_batch": U, "union_per_layer": u_stack or None,
            "int4_bytes_per_step": bytes_step, "int4_gbs": int4_gbs, "int4_frac_of_hbm": int4_gbs / hbm,
            "roofline": roof, "stage_ms": stage_ms,
            "cpu_baseline": cpu, "e2e": e2e, "e2e_eager": e2e_eager, "e2e_copies": e2e_copies, "tier": tier,
            "gpu_launches": launches, "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
