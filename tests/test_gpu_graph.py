"""The layer call is graph-capturable: it only enqueues work on the caller's
stream (no host synchronisation, no allocation), so a CUDA graph captured
around it and replayed on new inputs gives the same bits as eager calls."""
import numpy as np
import pytest
import torch

import synth
from tests._gpu import bits, device_layer, needs_gpu, to_dev_bits
from tests.test_gpu_parity import _small_shape, _status, lib  # noqa: F401

pytestmark = [pytest.mark.gpu, needs_gpu]


@pytest.mark.parametrize("T,flags", [(1, 0), (4, 0x1), (8, 0x10), (40, 0x20)],
                         ids=["b1", "b4-prenorm", "b8-decode-form", "b40-prefill-form"])
def test_layer_replays_from_a_cuda_graph(lib, T, flags):
    shape = _small_shape(tokens=T, n_shared=1)
    layer = device_layer(shape, seed=13)
    xs = [synth.normal_bf16(13, 20 + b, synth.X_IN, (T, shape.hidden)) for b in range(3)]
    ws = layer.workspace(T)
    # eager results (also warms the library's per-device state before capture)
    eager = []
    for xb in xs:
        x = to_dev_bits(xb)
        out = torch.empty_like(x)
        layer.forward(x, out, ws, residual=x, flags=flags)
        eager.append(bits(out))
    assert _status(lib) == 0
    x_static = to_dev_bits(xs[0])
    out_static = torch.empty_like(x_static)
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        layer.forward(x_static, out_static, ws, residual=x_static, flags=flags)
    for xb, want in zip(xs, eager):
        x_static.copy_(to_dev_bits(xb))
        g.replay()
        torch.cuda.synchronize()
        assert np.array_equal(bits(out_static), want)
    assert _status(lib) == 0
