"""Host-RAM expert tier (coli_moe_layer_tiered, coli_moe_tier_prefetch).

Placement changes where an expert is read from, never what the layer
computes: every tiered call's output must equal the all-resident layer's bit
for bit, in the split-K and the two-phase decode forms, over sequences of
calls that hit, miss and evict.  The tier's state after each call must equal
a plain model of the documented policy (hits stamped first; each miss, in the
union's order, into the first slot of the eviction order: empty, then least
routed, then least recently used, then lowest index; usage += routed pairs),
and every occupied slot must hold its expert's bytes.  A prefetch places
experts without counting them, and a following call that routes to them has
no miss.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import synth.gpu as sg
from tests._gpu import bits, device_layer, needs_gpu, to_dev_bits

pytestmark = [pytest.mark.gpu, needs_gpu]

NAMES = ("gate_q", "up_q", "down_q", "gate_s", "up_s", "down_s")


@pytest.fixture(scope="module")
def m():
    import int4_routed_expert_renorm_b200 as cm
    cm.coli_moe_get_status()
    return cm


class PolicyModel:
    """The placement policy of the header, step by step in Python."""

    def __init__(self, E, C):
        self.E, self.C = E, C
        self.slot_of = np.full(E, -1, np.int64)
        self.owner = np.full(C, -1, np.int64)
        self.usage = np.zeros(E, np.int64)
        self.last = np.zeros(C, np.int64)
        self.calls = self.hits = self.misses = self.fills = 0

    def _victim(self):
        best = None
        for c in range(self.C):
            if self.owner[c] >= 0 and self.last[c] == self.calls:
                continue
            key = (0,) if self.owner[c] < 0 else (1, min(int(self.usage[self.owner[c]]), 2 ** 31 - 1),
                                                  int(self.last[c]))
            if best is None or (key, c) < best:
                best = (key, c)
        return best[1]

    def place(self, ids, counts=None):
        self.calls += 1
        for e in ids:
            if self.slot_of[e] >= 0:
                self.last[self.slot_of[e]] = self.calls
        n_miss = 0
        for e in ids:
            if self.slot_of[e] >= 0:
                continue
            v = self._victim()
            if self.owner[v] >= 0:
                self.slot_of[self.owner[v]] = -1
            self.owner[v], self.slot_of[e], self.last[v] = e, v, self.calls
            n_miss += 1
        self.fills += n_miss
        if counts is not None:
            self.hits += len(ids) - n_miss
            self.misses += n_miss
            for e, cnt in zip(ids, counts):
                self.usage[e] += cnt

    def check(self, st):
        assert np.array_equal(st["slot_of"], self.slot_of)
        assert np.array_equal(st["owner"], self.owner)
        assert np.array_equal(st["usage"], self.usage)
        assert np.array_equal(st["last"], self.last)
        assert (st["calls"], st["hits"], st["misses"], st["fills"]) == (self.calls, self.hits, self.misses,
                                                                        self.fills)


def _setup(m, T_max, E, k, C, seed):
    shape = synth.LayerShape(f"tier_e{E}_k{k}", 512, 512, E, k, 1, T_max)
    full = sg.expert_tensors(shape, seed)
    li = synth.LayerInputs(shape, seed)
    rw = torch.from_numpy(li.router_w()).cuda()
    b = li.bias()
    bias = None if b is None else torch.from_numpy(b).cuda()
    resident = device_layer(shape, seed=seed)
    tl = m.tier.TieredLayer(resident.dims, full, C, rw, bias)
    return shape, full, resident, tl


def _logits(rng, T, E, skew):
    # a skewed router: low-index experts come up more often, so calls both
    # hit and miss
    return (rng.standard_normal((T, E)) + skew * np.linspace(1.0, 0.0, E)[None, :]).astype(np.float32)


@pytest.mark.parametrize("E,k,C,Ts", [(32, 2, 10, [1, 2, 5, 1, 3, 4, 2, 5, 1, 4]),
                                      (32, 2, 20, [9, 10, 9, 10, 9])],
                         ids=["split-K", "two-phase"])
def test_tier_matches_resident_layer_and_policy(m, E, k, C, Ts):
    shape, full, resident, tl = _setup(m, max(Ts), E, k, C, seed=41)
    rng = np.random.default_rng(41)
    model = PolicyModel(E, C)
    ws_r, ws_t = resident.workspace(max(Ts)), tl.workspace(max(Ts))
    for i, T in enumerate(Ts):
        l32 = _logits(rng, T, E, 2.0)
        x = synth.normal_bf16(41, 100 + i, synth.X_IN, (T, 512))
        xd, lg = to_dev_bits(x), torch.from_numpy(l32).cuda()
        o_r, o_t = torch.empty_like(xd), torch.empty_like(xd)
        ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
        resident.forward(xd, o_r, ws_r, logits_in=lg, residual=xd)
        tl.forward(xd, o_t, ws_t, logits_in=lg, residual=xd, topk_ids_out=ids)
        st_, fl = m.coli_moe_get_status()
        assert st_ == 0 and fl == 0
        assert np.array_equal(bits(o_t), bits(o_r)), f"call {i} (T={T})"
        gid = ids.cpu().numpy()
        assert np.array_equal(gid, oracle.route(l32, k)[0])
        u, seg, _, _ = oracle.batch_union(gid, E)
        model.place(u.tolist(), np.diff(seg).tolist())
        model.check(tl.state_arrays())
    assert model.hits > 0 and model.misses > C          # the sequence both hit and evicted
    # every occupied slot holds its expert's bytes
    owner = tl.state_arrays()["owner"]
    for c, e in enumerate(owner):
        if e >= 0:
            for name in NAMES:
                assert torch.equal(tl.slots[name][c], full[name][e].to(tl.slots[name].device)), (name, c, e)
    del full, resident, tl
    torch.cuda.empty_cache()


def test_tier_prefetch_places_without_counting(m):
    E, k, C, T = 32, 2, 8, 2
    shape, full, resident, tl = _setup(m, T, E, k, C, seed=42)
    want = torch.tensor([5, 17, 5, 30, 2], dtype=torch.int32, device="cuda")   # a repeat included
    tl.prefetch(want)
    st = tl.state_arrays()
    assert st["calls"] == 1 and st["hits"] == 0 and st["misses"] == 0 and st["fills"] == 4
    assert all(st["slot_of"][e] >= 0 for e in (5, 17, 30, 2)) and st["usage"].sum() == 0
    # a call that routes every token to prefetched experts misses nothing
    l32 = np.full((T, E), -5.0, np.float32)
    l32[0, 5], l32[0, 17], l32[1, 30], l32[1, 2] = 3.0, 2.0, 3.0, 2.0
    x = synth.normal_bf16(42, 5, synth.X_IN, (T, 512))
    xd, lg = to_dev_bits(x), torch.from_numpy(l32).cuda()
    o_t, o_r = torch.empty_like(xd), torch.empty_like(xd)
    tl.forward(xd, o_t, tl.workspace(T), logits_in=lg)
    resident.forward(xd, o_r, resident.workspace(T), logits_in=lg)
    st = tl.state_arrays()
    assert st["misses"] == 0 and st["hits"] == 4 and st["fills"] == 4
    assert np.array_equal(bits(o_t), bits(o_r))
    assert st["usage"][[5, 17, 30, 2]].tolist() == [1, 1, 1, 1]
    del full, resident, tl
    torch.cuda.empty_cache()


def test_tier_refuses_what_it_cannot_hold(m):
    E, k, C = 32, 2, 4
    shape, full, resident, tl = _setup(m, 40, E, k, C, seed=43)
    x = to_dev_bits(synth.normal_bf16(43, 5, synth.X_IN, (3, 512)))
    o = torch.empty_like(x)
    ws = tl.workspace(40)
    with pytest.raises(m.ColiError) as ei:          # min(E, T*k) = 6 > 4 slots
        tl.forward(x, o, ws)
    assert ei.value.status == m._lib.COLI_ERR_UNSUPPORTED
    x2 = to_dev_bits(synth.normal_bf16(43, 6, synth.X_IN, (2, 512)))
    with pytest.raises(m.ColiError) as ei:          # the prefill form is not tiered
        tl.forward(x2, torch.empty_like(x2), ws, flags=m._lib.COLI_PATH_PREFILL)
    assert ei.value.status == m._lib.COLI_ERR_UNSUPPORTED
    with pytest.raises(m.ColiError):                # more ids than slots
        tl.prefetch(torch.arange(5, dtype=torch.int32, device="cuda"))
    st_, fl = m.coli_moe_get_status()
    assert st_ == 0 and fl == 0
    del full, resident, tl
    torch.cuda.empty_cache()


def test_tier_warm_start_from_a_usage_profile(m):
    """Learn across runs: a saved usage profile makes its most used experts
    resident before the first call (the pages' pinned hot experts), and the
    counts carry on from it."""
    E, k, C = 32, 2, 6
    shape, full, resident, tl = _setup(m, 2, E, k, C, seed=44)
    profile = np.zeros(E, np.int64)
    profile[[3, 9, 10, 21, 30, 31, 7]] = [50, 40, 40, 30, 20, 20, 20]   # 31 and 7 tie with 30: lower index wins
    tl.warm_from_usage(profile)
    st = tl.state_arrays()
    assert sorted(st["owner"].tolist()) == [3, 7, 9, 10, 21, 30]
    assert np.array_equal(st["usage"], profile.astype(np.uint32))
    # a call that routes to two of them hits and adds its pairs to the profile
    T = 1
    l32 = np.full((T, E), -5.0, np.float32)
    l32[0, 9], l32[0, 21] = 2.0, 1.0
    x = synth.normal_bf16(44, 5, synth.X_IN, (T, 512))
    xd, lg = to_dev_bits(x), torch.from_numpy(l32).cuda()
    o_t, o_r = torch.empty_like(xd), torch.empty_like(xd)
    tl.forward(xd, o_t, tl.workspace(T), logits_in=lg)
    resident.forward(xd, o_r, resident.workspace(T), logits_in=lg)
    st = tl.state_arrays()
    assert st["hits"] == 2 and st["misses"] == 0
    assert st["usage"][9] == 41 and st["usage"][21] == 31
    assert np.array_equal(bits(o_t), bits(o_r))
    del full, resident, tl
    torch.cuda.empty_cache()


def test_tier_lookahead_places_the_next_layers_experts(m):
    """Overlap: routing a layer's input with the next layer's router on a side
    stream places that layer's experts while the current one runs; when the
    next layer then sees the same rows it routes them identically and misses
    nothing."""
    E, k, C, T = 32, 2, 8, 3
    shape, full, resident, cur = _setup(m, T, E, k, C, seed=45)
    shape2, full2, resident2, nxt = _setup(m, T, E, k, C, seed=46)
    x = synth.normal_bf16(45, 5, synth.X_IN, (T, 512))
    xd = to_dev_bits(x)
    o_cur = torch.empty_like(xd)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    ws_side = nxt.workspace(T)
    with torch.cuda.stream(side):
        nxt.lookahead(xd, ws_side, stream=side)
    cur.forward(xd, o_cur, cur.workspace(T))           # the current layer meanwhile
    torch.cuda.current_stream().wait_stream(side)
    st = nxt.state_arrays()
    assert st["fills"] > 0 and st["hits"] == 0 and st["misses"] == 0 and st["usage"].sum() == 0
    o_t, o_r = torch.empty_like(xd), torch.empty_like(xd)
    nxt.forward(xd, o_t, nxt.workspace(T))
    resident2.forward(xd, o_r, resident2.workspace(T))
    st = nxt.state_arrays()
    assert st["misses"] == 0 and st["hits"] > 0
    assert np.array_equal(bits(o_t), bits(o_r))
    s_, fl = m.coli_moe_get_status()
    assert s_ == 0 and fl == 0
    del full, resident, cur, full2, resident2, nxt
    torch.cuda.empty_cache()
