"""Host-memory input and output (COLI_LAYER_HOST_X, COLI_LAYER_HOST_OUT).

With the flags, coli_moe_layer reads x (and the residual) from page-locked
host memory through one staging kernel and writes out straight into
page-locked host memory from its last kernel.  The layer's arithmetic is the
same, so the outputs must equal the device-buffer call's bit for bit, in
every FFN form (split-K decode with the routing kernel and with its own
routing, two-phase decode, prefill), with and without a residual, with
pre-norm, inside a CUDA graph, and through the allocation-free entry.
Pointers the device cannot reach are refused before anything launches.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
from tests._gpu import bits, device_layer, needs_gpu, to_dev_bits

pytestmark = [pytest.mark.gpu, needs_gpu]


@pytest.fixture(scope="module")
def m():
    import int4_routed_expert_renorm_b200 as cm
    cm.coli_moe_get_status()
    return cm


def _shape(T):
    return synth.LayerShape(f"hostio_t{T}", 512, 512, 16, 4, 1, T)


def _pinned_bits(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).pin_memory()


@pytest.mark.parametrize("T,flags,res", [(1, 0, None), (4, 0, "x"), (6, 0x1, "x"), (40, 0, "other"),
                                         (64, 0x20, "x"), (3, 0x10, "other")],
                         ids=["T1-splitk", "T4-splitk-own-routing", "T6-prenorm", "T40-two-phase",
                              "T64-prefill", "T3-residual"])
def test_host_io_matches_device_buffers(m, T, flags, res):
    shape = _shape(T)
    layer = device_layer(shape, seed=31)
    x = synth.normal_bf16(31, 5, synth.X_IN, (T, 512))
    r = None if res is None else (x if res == "x" else synth.normal_bf16(31, 6, synth.X_IN, (T, 512)))
    # the device-buffer call
    xd = to_dev_bits(x)
    rd = None if r is None else (xd if res == "x" else to_dev_bits(r))
    od = torch.empty_like(xd)
    layer.forward(xd, od, layer.workspace(T), residual=rd, flags=flags)
    # the same through host memory
    xh = _pinned_bits(x)
    rh = None if r is None else (xh if res == "x" else _pinned_bits(r))
    oh = torch.zeros_like(xh).pin_memory()
    ws = layer.workspace(T)
    layer.forward(xh, oh, ws, residual=rh, flags=flags | m._lib.COLI_LAYER_HOST_X | m._lib.COLI_LAYER_HOST_OUT)
    torch.cuda.synchronize()
    st, fl = m.coli_moe_get_status()
    assert st == 0 and fl == 0
    assert np.array_equal(oh.numpy().view(np.uint16), bits(od))


def test_host_io_in_a_graph_and_without_allocation(m):
    T = 2
    shape = _shape(T)
    layer = device_layer(shape, seed=32)
    xs = [synth.normal_bf16(32, 5 + b, synth.X_IN, (T, 512)) for b in range(2)]
    refs = []
    for x in xs:
        xd = to_dev_bits(x)
        od = torch.empty_like(xd)
        layer.forward(xd, od, layer.workspace(T))
        refs.append(bits(od))
    flags = m._lib.COLI_LAYER_HOST_X | m._lib.COLI_LAYER_HOST_OUT
    xh = _pinned_bits(xs[0])
    oh = torch.zeros_like(xh).pin_memory()
    ws = layer.workspace(T)
    layer.forward(xh, oh, ws, flags=flags)           # first call outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g):
            layer.forward(xh, oh, ws, flags=flags)
    torch.cuda.current_stream().wait_stream(s)
    for x, ref in zip(xs, refs):
        xh.copy_(torch.from_numpy(np.ascontiguousarray(x).view(np.int16)))   # new input in place
        g.replay()
        torch.cuda.synchronize()
        assert np.array_equal(oh.numpy().view(np.uint16), ref)
    oh.zero_()
    m.coli_moe_layer_noalloc(layer.dims, layer.weights, xh, oh, flags=flags)
    torch.cuda.synchronize()
    assert np.array_equal(oh.numpy().view(np.uint16), refs[1])
    st, fl = m.coli_moe_get_status()
    assert st == 0 and fl == 0


def test_host_flags_refuse_unreachable_or_device_pointers(m):
    T = 1
    shape = _shape(T)
    layer = device_layer(shape, seed=33)
    lib = m._lib._lib
    d, w = layer.dims, layer.weights
    ws = layer.workspace(T)
    n = ws.numel()
    x_pageable = np.zeros((T, 512), np.int16)                    # ordinary (pageable) host memory
    out_dev = torch.empty((T, 512), dtype=torch.int16, device="cuda")
    x_dev = torch.zeros((T, 512), dtype=torch.int16, device="cuda")
    hx, ho = m._lib.COLI_LAYER_HOST_X, m._lib.COLI_LAYER_HOST_OUT

    def call(x_ptr, out_ptr, flags):
        return lib.coli_moe_layer(ctypes.byref(d), ctypes.byref(w), x_ptr, T, None, None, flags, out_ptr, None, None,
                                  None, ctypes.c_void_p(ws.data_ptr()), n, None)

    px = ctypes.c_void_p(x_pageable.ctypes.data)
    assert call(px, ctypes.c_void_p(out_dev.data_ptr()), hx) == m._lib.COLI_ERR_INVALID_ARG
    # a device pointer under the host flags is refused as well
    assert call(ctypes.c_void_p(x_dev.data_ptr()), ctypes.c_void_p(out_dev.data_ptr()), hx) == m._lib.COLI_ERR_INVALID_ARG
    assert call(ctypes.c_void_p(x_dev.data_ptr()), ctypes.c_void_p(out_dev.data_ptr()), ho) == m._lib.COLI_ERR_INVALID_ARG
    # the binding refuses a CPU tensor that is not page-locked
    with pytest.raises(ValueError, match="page-locked"):
        layer.forward(torch.zeros((T, 512), dtype=torch.int16), out_dev, ws, flags=hx)
    torch.cuda.synchronize()
    st, fl = m.coli_moe_get_status()
    assert st == 0 and fl == 0
