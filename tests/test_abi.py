"""The C-ABI library loads, exports every symbol include/*.h declares, and its
host-side argument checks answer before anything is launched.  CPU only: no
call here reaches a kernel launch."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        for m in re.finditer(r"\b(coli_[a-z0-9_]+)\s*\(", src):
            names.add(m.group(1))
    return names


@pytest.fixture(scope="module")
def colimoe():
    from int4_routed_expert_renorm_b200.build import build
    build()
    import int4_routed_expert_renorm_b200 as m
    return m


def test_every_declared_symbol_is_exported(colimoe):
    lib = ctypes.CDLL(colimoe._lib.LIB_PATH)
    declared = _declared_functions()
    assert {"coli_moe_route", "coli_moe_union", "coli_moe_expert_ffn", "coli_moe_layer"} <= declared
    missing = [n for n in sorted(declared) if not hasattr(lib, n)]
    assert not missing, missing
    assert set(colimoe._lib.EXPORTS) <= declared


def test_version_and_status_strings(colimoe):
    assert colimoe.coli_moe_version() >= 100
    assert colimoe._lib.status_str(0) == "ok"
    assert colimoe._lib.status_str(3) == "workspace too small"


def _dims(m, **kw):
    d = dict(hidden=6144, inter=2048, n_experts=256, top_k=8, n_shared=1, group=32, code_bits=4)
    d.update(kw)
    return m.coli_moe_dims(**d)


def test_workspace_bytes(colimoe):
    m = colimoe
    d = _dims(m)
    n1 = m.coli_moe_workspace_bytes(d, 1)
    n64 = m.coli_moe_workspace_bytes(d, 64)
    assert 0 < n1 < n64
    # ypair rows (T*k + S*T) x H fp32 dominate: at least that much
    assert n64 >= (64 * 8 + 64) * 6144 * 4
    assert m.coli_moe_workspace_bytes(_dims(m, group=64), 4) == m.coli_moe_workspace_bytes(d, 4)
    assert m.coli_moe_workspace_bytes(_dims(m, group=16), 4) == 0
    assert m.coli_moe_workspace_bytes(_dims(m, group=128), 4) == 0
    # group 64 reads scales in boxes of 8 (512 codes): H and I multiples of 512
    assert m.coli_moe_workspace_bytes(_dims(m, group=64, hidden=6400), 4) == 0
    assert m.coli_moe_workspace_bytes(_dims(m, group=64, inter=768), 4) == 0
    assert m.coli_moe_workspace_bytes(_dims(m, group=32, hidden=6400, inter=768), 4) > 0
    # int8 codes (code_bits 8): the split-K decode form needs whole 16-byte down scale rows
    assert m.coli_moe_workspace_bytes(_dims(m, code_bits=8), 4) == m.coli_moe_workspace_bytes(d, 4)
    assert m.coli_moe_workspace_bytes(_dims(m, code_bits=8, inter=128), 4) == 0
    assert m.coli_moe_workspace_bytes(_dims(m, code_bits=5), 4) == 0
    assert m.coli_moe_workspace_bytes(_dims(m, hidden=6000), 4) == 0
    assert m.coli_moe_workspace_bytes(_dims(m, top_k=300), 4) == 0


def _fake(addr=0x10000):
    return ctypes.c_void_p(addr)


def test_route_and_union_argument_checks(colimoe):
    lib = colimoe._lib._lib
    f = _fake()
    assert lib.coli_moe_route(f, None, 4, 2000, 8, f, f, None) == colimoe._lib.COLI_ERR_UNSUPPORTED
    assert lib.coli_moe_route(f, None, 4, 16, 17, f, f, None) == colimoe._lib.COLI_ERR_UNSUPPORTED
    assert lib.coli_moe_route(None, None, 4, 16, 2, f, f, None) == colimoe._lib.COLI_ERR_INVALID_ARG
    assert lib.coli_moe_route(f, None, -1, 16, 2, f, f, None) == colimoe._lib.COLI_ERR_INVALID_ARG
    assert lib.coli_moe_route(None, None, 0, 16, 2, None, None, None) == colimoe._lib.COLI_OK  # T = 0: no-op
    assert lib.coli_moe_union(f, 4, 2, 2000, f, f, f, f, f, None) == colimoe._lib.COLI_ERR_UNSUPPORTED
    assert lib.coli_moe_union(f, 1 << 22, 8, 256, f, f, f, f, f, None) == colimoe._lib.COLI_ERR_UNSUPPORTED
    assert lib.coli_moe_union(f, 4, 2, 16, f, None, f, f, f, None) == colimoe._lib.COLI_ERR_INVALID_ARG


def _weights(m, misalign=False):
    a = 0x100000
    ptrs = [a + i * 0x1000 for i in range(8)]
    if misalign:
        ptrs[0] += 2
    return m.coli_moe_weights(*[ctypes.c_void_p(p) for p in ptrs])


def test_layer_argument_checks(colimoe):
    m = colimoe
    lib = m._lib._lib
    d, w = _dims(m), _weights(m)
    x, out, ws = _fake(0x200000), _fake(0x300000), _fake(0x400000)
    need = m.coli_moe_workspace_bytes(d, 4)
    L = lambda d_, w_, x_, T, ws_, nbytes, flags=0: lib.coli_moe_layer(  # noqa: E731
        ctypes.byref(d_), ctypes.byref(w_), x_, T, None, None, flags, out, None, None, None, ws_, nbytes, None)
    assert L(d, w, x, 4, ws, need - 1) == m._lib.COLI_ERR_WORKSPACE
    assert L(_dims(m, group=16), w, x, 4, ws, need) == m._lib.COLI_ERR_UNSUPPORTED
    assert L(_dims(m, group=64, inter=1280), w, x, 4, ws, need) == m._lib.COLI_ERR_UNSUPPORTED
    # int8 above 8 tokens: 8-token passes (past the checks a machine without a GPU stops at the device query)
    assert L(_dims(m, code_bits=8), w, x, 9, ws, m.coli_moe_workspace_bytes(d, 9)) in (m._lib.COLI_OK,
                                                                                      m._lib.COLI_ERR_CUDA)
    assert L(_dims(m, code_bits=8), w, x, 9, ws, m.coli_moe_workspace_bytes(d, 8) - 256) == m._lib.COLI_ERR_WORKSPACE
    assert L(_dims(m, code_bits=8), w, x, 4, ws, need, 0x20) == m._lib.COLI_ERR_UNSUPPORTED   # forced prefill
    assert L(_dims(m, inter=384), w, x, 4, ws, need) == m._lib.COLI_ERR_UNSUPPORTED
    assert L(_dims(m, n_shared=9), w, x, 4, ws, need) == m._lib.COLI_ERR_UNSUPPORTED
    assert L(d, _weights(m, misalign=True), x, 4, ws, need) == m._lib.COLI_ERR_INVALID_ARG
    assert L(d, w, None, 4, ws, need) == m._lib.COLI_ERR_INVALID_ARG
    assert L(d, w, x, 4, _fake(0x400010), need) == m._lib.COLI_ERR_INVALID_ARG   # ws not 256-aligned
    assert L(d, w, x, -2, ws, need) == m._lib.COLI_ERR_INVALID_ARG
    assert L(d, w, x, 0, ws, 0) == m._lib.COLI_OK                                # T = 0: no-op
    nw = m.coli_moe_weights(*[ctypes.c_void_p(0x100000 + i * 0x1000) for i in range(6)], None, None)
    assert L(d, nw, x, 4, ws, need) == m._lib.COLI_ERR_INVALID_ARG              # no router, no logits_in
    # host-memory flags: pointers the device cannot reach as host memory are refused
    assert L(d, w, x, 4, ws, need, m._lib.COLI_LAYER_HOST_X) == m._lib.COLI_ERR_INVALID_ARG
    assert L(d, w, x, 4, ws, need, m._lib.COLI_LAYER_HOST_OUT) == m._lib.COLI_ERR_INVALID_ARG


def test_expert_ffn_argument_checks(colimoe):
    m = colimoe
    lib = m._lib._lib
    d, w, f = _dims(m), _weights(m), _fake(0x500000)
    need = m.coli_moe_workspace_bytes(d, 4)
    F = lambda T, ws_bytes, x=f, out=_fake(0x600000): lib.coli_moe_expert_ffn(  # noqa: E731
        ctypes.byref(d), ctypes.byref(w), x, T, f, f, f, f, f, f, f, None, out, 0, _fake(0x700000), ws_bytes, None)
    assert F(4, need - 256) == m._lib.COLI_ERR_WORKSPACE
    assert F(4, need, x=_fake(0x600000)) == m._lib.COLI_ERR_INVALID_ARG   # out aliases x
    assert F(0, 0) == m._lib.COLI_OK
    for hf in (m._lib.COLI_LAYER_HOST_X, m._lib.COLI_LAYER_HOST_OUT):         # device buffers only
        assert lib.coli_moe_expert_ffn(ctypes.byref(d), ctypes.byref(w), f, 4, f, f, f, f, f, f, f, None,
                                       _fake(0x600000), hf, _fake(0x700000), need, None) == m._lib.COLI_ERR_UNSUPPORTED


def test_tier_state_bytes_and_argument_checks(colimoe):
    """The tier's state size (int32 words: 2 E + 4 C + 5, 256-byte aligned)
    and the checks that need no GPU."""
    m = colimoe
    lib = m._lib._lib
    d = _dims(m)
    E = d.n_experts
    for C in (1, 7, E):
        assert m.coli_moe_tier_state_bytes(d, C) == -(-(4 * (2 * E + 4 * C + 5)) // 256) * 256
    assert m.coli_moe_tier_state_bytes(d, 0) == 0 and m.coli_moe_tier_state_bytes(d, E + 1) == 0
    f = ctypes.c_void_p(0x10000)
    t = m.coli_moe_tier(f, f, f, f, f, f, 4, ctypes.c_void_p(0x20000))
    assert lib.coli_moe_tier_reset(ctypes.byref(d), ctypes.byref(m.coli_moe_tier(f, f, f, f, f, f, 0, f)),
                                   None) == m._lib.COLI_ERR_INVALID_ARG       # no slots
    assert lib.coli_moe_tier_reset(ctypes.byref(d), ctypes.byref(m.coli_moe_tier(f, f, f, f, f, f, 4,
                                                                                 ctypes.c_void_p(0x20010))),
                                   None) == m._lib.COLI_ERR_INVALID_ARG       # state not 256-byte aligned
    w = _weights(m)
    # host arrays the device cannot reach as host memory are refused
    assert lib.coli_moe_tier_prefetch(ctypes.byref(d), ctypes.byref(w), ctypes.byref(t), f, 2,
                                      None) == m._lib.COLI_ERR_INVALID_ARG
    x, out, ws = _fake(0x200000), _fake(0x300000), _fake(0x400000)
    assert lib.coli_moe_layer_tiered(ctypes.byref(d), ctypes.byref(w), ctypes.byref(t), x, 1, None, None, 0, out,
                                     None, None, None, ws, m.coli_moe_workspace_bytes(d, 1),
                                     None) == m._lib.COLI_ERR_INVALID_ARG
    assert lib.coli_moe_tier_lookahead(ctypes.byref(d), ctypes.byref(w), ctypes.byref(t), x, 1, 0, ws,
                                       m.coli_moe_workspace_bytes(d, 1), None) == m._lib.COLI_ERR_INVALID_ARG
    assert lib.coli_moe_tier_lookahead(ctypes.byref(d), ctypes.byref(w),
                                       ctypes.byref(m.coli_moe_tier(f, f, f, f, f, f, 0, f)), x, 1, 0, ws,
                                       m.coli_moe_workspace_bytes(d, 1), None) == m._lib.COLI_ERR_INVALID_ARG


def test_binding_host_flags_need_page_locked_tensors(colimoe):
    """Under COLI_LAYER_HOST_X the binding passes x (and the residual) only as
    page-locked CPU tensors; anything else is refused before the library."""
    import torch
    m = colimoe
    d, w = _dims(m), _weights(m)
    x = torch.zeros(2, d.hidden, dtype=torch.int16)            # CPU, not page-locked
    with pytest.raises(ValueError, match="page-locked"):
        m._lib.coli_moe_layer(d, w, x, torch.zeros_like(x), torch.empty(16, dtype=torch.uint8),
                              flags=m._lib.COLI_LAYER_HOST_X)


def test_binding_fails_loudly_without_library(tmp_path):
    from int4_routed_expert_renorm_b200 import _lib
    with pytest.raises(ImportError):
        _lib.load(str(tmp_path / "libcolimoe.so"))


def test_binding_constants_match_the_header(colimoe):
    """Every #define of the header that the binding mirrors has the same value."""
    src = open(os.path.join(ROOT, "include", "coli_moe.h")).read()
    found = 0
    for m in re.finditer(r"#define\s+(COLI_[A-Z_]+)\s+\(?(0x[0-9a-fA-F]+|\d+)u?(?:\s*<<\s*(\d+))?\)?", src):
        name, val, sh = m.group(1), int(m.group(2), 0), m.group(3)
        if sh:
            val <<= int(sh)
        if hasattr(colimoe._lib, name):
            assert getattr(colimoe._lib, name) == val, name
            found += 1
    assert found >= 7


def _form_rule(T, E, k, inter=2048, code_bits=4, flags=0):
    """The dispatch rule as include/coli_moe.h states it (COLI_PATH_* and
    COLI_FORM_* comments)."""
    fd, fp = bool(flags & 0x10), bool(flags & 0x20)
    if T == 0:
        return 0          # a no-op call, whatever the flags
    if fd and fp:
        return "invalid"
    splitk = T <= 8 and inter % 256 == 0
    if code_bits == 8:   # the split-K form, batches above 8 tokens in 8-token passes
        return 1 if (inter % 256 == 0 and not fp) else "unsupported"
    P = T * k
    prefill = fp or (not fd and T >= 32 and P >= 32 * min(E, P))
    return 3 if prefill else (1 if splitk else 2)


def test_ffn_form_follows_the_documented_rule(colimoe):
    m = colimoe
    errs = {m._lib.COLI_ERR_INVALID_ARG: "invalid", m._lib.COLI_ERR_UNSUPPORTED: "unsupported"}

    def form(T, flags=0, **kw):
        try:
            return m.coli_moe_ffn_form(_dims(m, **kw), T, flags)
        except m._lib.ColiError as e:
            return errs[e.status]

    for E, k in ((8, 1), (16, 2), (64, 8), (256, 8)):
        for T in list(range(0, 70)) + [255, 256, 257, 511, 512, 1023, 1024, 1025, 4096]:
            for flags in (0, 0x10, 0x20, 0x30):
                assert form(T, flags, n_experts=E, top_k=k) == _form_rule(T, E, k, flags=flags), (E, k, T, flags)
    for T in (1, 4, 8, 9, 64):
        for flags in (0, 0x10, 0x20):
            assert form(T, flags, inter=128) == _form_rule(T, 256, 8, inter=128, flags=flags)
            assert form(T, flags, code_bits=8) == _form_rule(T, 256, 8, code_bits=8, flags=flags)
    # the named cases: batch 1 splits K, batch 64 runs two phases, prefill 4096 takes tcgen05
    assert (form(1), form(64), form(4096)) == (m._lib.COLI_FORM_DECODE_SPLITK, m._lib.COLI_FORM_DECODE_TWOPHASE,
                                               m._lib.COLI_FORM_PREFILL)
    assert form(-1) == "invalid" and form(4, group=16) == "unsupported" and form(1 << 22) == "unsupported"
    lib, out = m._lib._lib, ctypes.c_int(7)
    assert lib.coli_moe_ffn_form(None, 4, 0, ctypes.byref(out)) == m._lib.COLI_ERR_INVALID_ARG and out.value == 0
    assert lib.coli_moe_ffn_form(ctypes.byref(_dims(m)), 4, 0, None) == m._lib.COLI_ERR_INVALID_ARG


def test_bench_form_helpers_match_the_library(colimoe):
    """bench.py picks each workload's roofline by the form it expects the
    library to take: the library agrees for every workload."""
    import bench
    import synth
    m = colimoe
    for shape in synth.WORKLOADS.values():
        d = m.dims_for(shape.hidden, shape.inter, shape.n_experts, shape.top_k, shape.n_shared, shape.group,
                       shape.bits)
        f = m.coli_moe_ffn_form(d, shape.tokens)
        assert bench.splitk_form(shape) == (f == m._lib.COLI_FORM_DECODE_SPLITK), shape.name
        assert bench.prefill_form(shape) == (f == m._lib.COLI_FORM_PREFILL), shape.name


def _kw_cases(fn):
    return next(list(mk.args[1]) for mk in fn.pytestmark if mk.name == "parametrize" and mk.args[0] == "kw")


def test_gpu_tests_exercise_the_form_they_name(colimoe):
    """The split-K and int8 parity cases take the split-K decode form and the
    two-phase invariance cases the two-phase form (read from the tests' own
    parametrisations, so a later edit cannot silently move them)."""
    import tests.test_gpu_int8 as i8
    import tests.test_gpu_splitk as sk
    from tests.test_gpu_parity import _small_shape
    m = colimoe

    def form(shape, flags=0):
        d = m.dims_for(shape.hidden, shape.inter, shape.n_experts, shape.top_k, shape.n_shared, shape.group,
                       shape.bits)
        return m.coli_moe_ffn_form(d, shape.tokens, flags)

    for kw in _kw_cases(sk.test_splitk_small_shapes):
        assert form(_small_shape(**kw)) == m._lib.COLI_FORM_DECODE_SPLITK, kw
    for kw in _kw_cases(i8.test_int8_small_shapes):
        assert form(_small_shape(bits=8, **kw)) == m._lib.COLI_FORM_DECODE_SPLITK, kw
    for inter in (256, 512):
        for T in (9, 64, 65):
            shape = _small_shape(tokens=T, hidden=512, inter=inter, n_experts=8, top_k=2, n_shared=1)
            assert form(shape) == m._lib.COLI_FORM_DECODE_TWOPHASE, (inter, T)
    # int8 batches above 8 tokens run the split-K form in 8-token passes
    assert form(_small_shape(bits=8, tokens=9, inter=256)) == m._lib.COLI_FORM_DECODE_SPLITK


@pytest.mark.parametrize("bits", [4, 8])
def test_layer_holder_checks_tensor_sizes(colimoe, bits):
    """MoELayer accepts tensors sized for its dims (int4 or int8 codes) and
    rejects a wrong size before any call; CPU tensors stand in for device ones."""
    import torch
    m = colimoe
    H, I, E, S, G = 256, 256, 4, 1, 64
    d = m.dims_for(H, I, E, 2, S, G, bits)
    n = E + S
    t = {"gate_q": torch.zeros(n, I, H * bits // 8, dtype=torch.uint8),
         "up_q": torch.zeros(n, I, H * bits // 8, dtype=torch.uint8),
         "down_q": torch.zeros(n, H, I * bits // 8, dtype=torch.uint8),
         "gate_s": torch.zeros(n, I, H // G, dtype=torch.int16), "up_s": torch.zeros(n, I, H // G, dtype=torch.int16),
         "down_s": torch.zeros(n, H, I // G, dtype=torch.int16)}
    layer = m.MoELayer(d, t)
    assert layer.weights.gate_q == t["gate_q"].data_ptr() and layer.weights.down_s == t["down_s"].data_ptr()
    assert layer.weights.router_w is None
    for name in t:
        bad = dict(t)
        bad[name] = t[name][:, :-1]
        with pytest.raises(ValueError, match=name):
            m.MoELayer(d, bad)


@pytest.mark.parametrize("kw", [dict(), dict(group=64), dict(code_bits=8), dict(hidden=1024, inter=512, n_experts=16),
                                dict(hidden=256, inter=128, n_experts=16, top_k=2, n_shared=0)],
                         ids=["glm", "glm_gs64", "glm_int8", "mid", "tiny_i128"])
def test_workspace_for_t_max_covers_every_smaller_batch(colimoe, kw):
    """A workspace of coli_moe_workspace_bytes(dims, T_max) bytes passes the
    library's own workspace check for every batch of up to T_max tokens, in
    the layer and the FFN call.  (On a machine without a GPU a call that passes
    its checks stops at the device query with COLI_ERR_CUDA, before any launch.)"""
    m = colimoe
    lib = m._lib._lib
    d, w = _dims(m, **kw), _weights(m)
    int8 = kw.get("code_bits") == 8
    f = _fake(0x500000)
    t_maxes = list(range(0, 40)) + [63, 64, 65, 77, 78, 100, 129, 300]
    for t_max in t_maxes:
        n = m.coli_moe_workspace_bytes(d, t_max)
        assert n > 0
        for T in range(0, t_max + 1):
            if int8 and T > 8:
                break
            st_layer = lib.coli_moe_layer(ctypes.byref(d), ctypes.byref(w), _fake(0x200000), T, None, None, 0,
                                          _fake(0x300000), None, None, None, _fake(0x400000), n, None)
            st_ffn = lib.coli_moe_expert_ffn(ctypes.byref(d), ctypes.byref(w), _fake(0x200000), T, f, f, f, f, f, f,
                                             f, None, _fake(0x600000), 0, _fake(0x700000), n, None)
            assert st_layer != m._lib.COLI_ERR_WORKSPACE and st_ffn != m._lib.COLI_ERR_WORKSPACE, (t_max, T)
            assert st_layer in (m._lib.COLI_OK, m._lib.COLI_ERR_CUDA), st_layer
    # and the size is not padded beyond the largest batch's need: one byte less fails for some T <= T_max
    for t_max in (1, 8, 9, 64, 300):
        n = m.coli_moe_workspace_bytes(d, t_max)
        if int8 and t_max > 8:
            continue
        worst = [T for T in range(1, t_max + 1)
                 if lib.coli_moe_layer(ctypes.byref(d), ctypes.byref(w), _fake(0x200000), T, None, None, 0,
                                       _fake(0x300000), None, None, None, _fake(0x400000), n - 1, None)
                 == m._lib.COLI_ERR_WORKSPACE]
        assert worst, t_max


def test_ffn_form_status_equals_the_calls_status(colimoe):
    """For any dims, T and flags, coli_moe_ffn_form fails exactly when the
    layer and FFN calls fail on them (same status); when it succeeds the calls
    get past every check (to the device query, COLI_ERR_CUDA without a GPU)."""
    from hypothesis import HealthCheck, given, settings
    from hypothesis import strategies as st
    m = colimoe
    lib = m._lib._lib
    w, f = _weights(m), _fake(0x500000)
    big = 1 << 40

    @settings(max_examples=400, deadline=None, derandomize=True, suppress_health_check=list(HealthCheck))
    @given(hidden=st.sampled_from([128, 256, 512, 768, 1024, 6144, 6000]),
           inter=st.sampled_from([64, 128, 256, 384, 512, 768, 2048]),
           n_experts=st.sampled_from([1, 2, 16, 256, 1024, 1025]), top_k=st.sampled_from([1, 2, 8, 32, 33]),
           n_shared=st.sampled_from([0, 1, 4, 5]), group=st.sampled_from([16, 32, 64, 128]),
           code_bits=st.sampled_from([0, 4, 5, 8]), T=st.sampled_from([-1, 0, 1, 5, 8, 9, 64, 300, 4096]),
           flags=st.sampled_from([0, 0x1, 0x10, 0x20, 0x30, 0x11, 0x21]))
    def check(hidden, inter, n_experts, top_k, n_shared, group, code_bits, T, flags):
        d = m.coli_moe_dims(hidden, inter, n_experts, top_k, n_shared, group, code_bits)
        form = ctypes.c_int(-1)
        st_form = lib.coli_moe_ffn_form(ctypes.byref(d), T, flags, ctypes.byref(form))
        st_layer = lib.coli_moe_layer(ctypes.byref(d), ctypes.byref(w), _fake(0x200000), T, None, None, flags,
                                      _fake(0x300000), None, None, None, _fake(0x400000), big, None)
        st_ffn = lib.coli_moe_expert_ffn(ctypes.byref(d), ctypes.byref(w), _fake(0x200000), T, f, f, f, f, f, f, f,
                                         None, _fake(0x600000), flags, _fake(0x700000), big, None)
        if st_form != m._lib.COLI_OK:
            assert st_layer == st_form and st_ffn == st_form, (st_form, st_layer, st_ffn)
            assert form.value == 0
        elif T == 0:
            assert st_layer == st_ffn == m._lib.COLI_OK and form.value == 0
        else:
            assert st_layer == st_ffn == m._lib.COLI_ERR_CUDA and form.value in (1, 2, 3)

    check()


def test_layer_holder_workspace_refuses_unsupported_dims(colimoe):
    import torch
    m = colimoe
    H, I, E, S = 256, 256, 4, 1

    def holder(group):
        t = {"gate_q": torch.zeros(E + S, I, H // 2, dtype=torch.uint8),
             "up_q": torch.zeros(E + S, I, H // 2, dtype=torch.uint8),
             "down_q": torch.zeros(E + S, H, I // 2, dtype=torch.uint8),
             "gate_s": torch.zeros(E + S, I, H // group, dtype=torch.int16),
             "up_s": torch.zeros(E + S, I, H // group, dtype=torch.int16),
             "down_s": torch.zeros(E + S, H, I // group, dtype=torch.int16)}
        return m.MoELayer(m.dims_for(H, I, E, 2, S, group), t)

    assert holder(32).workspace(4, device="cpu").numel() == m.coli_moe_workspace_bytes(holder(32).dims, 4)
    with pytest.raises(m._lib.ColiError) as e:
        holder(16).workspace(4, device="cpu")
    assert e.value.status == m._lib.COLI_ERR_UNSUPPORTED
    with pytest.raises(m._lib.ColiError) as e:
        holder(32).workspace(-1, device="cpu")
    assert e.value.status == m._lib.COLI_ERR_INVALID_ARG


def test_binding_refuses_host_and_strided_tensors(colimoe):
    """Tensor arguments must be contiguous device buffers: a host tensor or a
    strided view is refused before anything reaches the library."""
    import torch
    m = colimoe
    lg = torch.zeros(4, 16)
    ids, w = torch.zeros(4, 2, dtype=torch.int32), torch.zeros(4, 2)
    with pytest.raises(ValueError, match="device memory"):
        m.coli_moe_route(lg, None, ids, w)
    with pytest.raises(ValueError, match="contiguous"):
        m.coli_moe_route(torch.zeros(16, 4).t(), None, ids, w)
    H, I, E, S, G = 256, 256, 4, 1, 32
    t = {"gate_q": torch.zeros(E + S, I, H // 2, dtype=torch.uint8),
         "up_q": torch.zeros(E + S, I, H // 2, dtype=torch.uint8),
         "down_q": torch.zeros(E + S, H, I // 2, dtype=torch.uint8),
         "gate_s": torch.zeros(E + S, I, H // G, dtype=torch.int16),
         "up_s": torch.zeros(E + S, I, H // G, dtype=torch.int16),
         "down_s": torch.zeros(E + S, H, I // G, dtype=torch.int16)}
    d = m.dims_for(H, I, E, 2, S, G)
    layer = m.MoELayer(d, t)                                  # host tensors are held, but never run
    x = torch.zeros(2, H, dtype=torch.int16)
    with pytest.raises(ValueError, match="device memory"):
        layer.forward(x, torch.empty_like(x), torch.empty(16, dtype=torch.uint8))
    bad = dict(t, down_s=torch.zeros(E + S, I // G, H, dtype=torch.int16).transpose(1, 2))
    with pytest.raises(ValueError, match="contiguous"):
        m.MoELayer(d, bad)


def test_binding_refuses_tensors_of_the_wrong_size(colimoe):
    """Every tensor argument must have exactly the elements (and element size)
    the C call reads or writes through its pointer: a short or mistyped tensor
    is refused with ValueError before anything reaches the library (these are
    host tensors, which would be refused later anyway; the size check comes
    first)."""
    import torch
    m = colimoe
    H, I, E, k, S, T = 256, 256, 8, 2, 1, 3
    d = m.dims_for(H, I, E, k, S)
    w = m.coli_moe_weights()
    x = torch.zeros(T, H, dtype=torch.int16)
    out = torch.zeros(T, H, dtype=torch.int16)
    ws = torch.zeros(16, dtype=torch.uint8)
    good = dict(logits_in=torch.zeros(T, E), residual=torch.zeros(T, H, dtype=torch.int16),
                logits_out=torch.zeros(T, E), topk_ids_out=torch.zeros(T, k, dtype=torch.int32),
                topk_w_out=torch.zeros(T, k))
    bad = dict(logits_in=torch.zeros(T, E - 1), residual=torch.zeros(T - 1, H, dtype=torch.int16),
               logits_out=torch.zeros(T, E, dtype=torch.float64), topk_ids_out=torch.zeros(T, k + 1, dtype=torch.int32),
               topk_w_out=torch.zeros(T * k - 1))
    for name in bad:
        kw = dict(good, **{name: bad[name]})
        with pytest.raises(ValueError, match=name):
            m.coli_moe_layer(d, w, x, out, ws, **kw)
        with pytest.raises(ValueError, match=name):
            m.coli_moe_layer_noalloc(d, w, x, out, **kw)
    with pytest.raises(ValueError, match="x"):
        m.coli_moe_layer(d, w, torch.zeros(T, H + 8, dtype=torch.int16), out, ws)
    with pytest.raises(ValueError, match="x"):
        m.coli_moe_layer(d, w, torch.zeros(T, H, dtype=torch.float32), out, ws)
    with pytest.raises(ValueError, match="out"):
        m.coli_moe_layer(d, w, x, torch.zeros(T, H - 1, dtype=torch.int16), ws)
    # expert FFN: the union arrays
    P, U = T * k, min(E, T * k)
    i32 = lambda n: torch.zeros(n, dtype=torch.int32)  # noqa: E731
    args = dict(topk_ids=i32(P), topk_w=torch.zeros(P), unique_ids=i32(U), n_unique=i32(1), seg_off=i32(U + 1),
                perm=i32(P), pair_pos=i32(P))
    for name, short in (("topk_ids", i32(P - 1)), ("topk_w", torch.zeros(P + 1)), ("unique_ids", i32(U - 1)),
                        ("n_unique", i32(0)), ("seg_off", i32(U)), ("perm", i32(P - 1)), ("pair_pos", i32(P - 1))):
        a = dict(args, **{name: short})
        with pytest.raises(ValueError, match=name):
            m.coli_moe_expert_ffn(d, w, x, a["topk_ids"], a["topk_w"], a["unique_ids"], a["n_unique"],
                                  a["seg_off"], a["perm"], a["pair_pos"], None, out, ws)
    # route and union
    lg, ids, tw = torch.zeros(T, E), torch.zeros(T, k, dtype=torch.int32), torch.zeros(T, k)
    with pytest.raises(ValueError, match="bias"):
        m.coli_moe_route(lg, torch.zeros(E - 1), ids, tw)
    with pytest.raises(ValueError, match="topk_w"):
        m.coli_moe_route(lg, None, ids, torch.zeros(T, k, dtype=torch.float16))
    with pytest.raises(ValueError, match="pair_pos"):
        m.coli_moe_union(ids, E, i32(U), i32(1), i32(U + 1), i32(P), i32(P - 1))
    with pytest.raises(ValueError, match="seg_off"):
        m.coli_moe_union(ids, E, i32(U), i32(1), i32(U), i32(P), i32(P))
