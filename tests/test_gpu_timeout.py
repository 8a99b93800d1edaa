"""The device-side bounded waits give up, report and return.

Every pipeline wait of the FFN kernels (mbarrier phases, the token-block and
grid-wide counters) polls %globaltimer and gives up after a limit (2 s in the
kernels), setting COLI_FLAG_TIMEOUT instead of hanging the GPU.  The test hook
coli_moe_test_wait_timeout runs the same two wait routines with a limit of a
few milliseconds on a barrier nothing arrives on and a counter nothing
increments.  Both must give up after about that long, the status word must
say so, and the device must then run a normal layer call that matches the
oracle.  No kernel traps and nothing is left waiting.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._gpu import OUT_REL_TOL, bits, device_layer, needs_gpu, oracle_weights, to_dev_bits

pytestmark = [pytest.mark.gpu, needs_gpu]


@pytest.fixture(scope="module")
def lib():
    import int4_routed_expert_renorm_b200 as m
    m.coli_moe_get_status()
    return m


@pytest.mark.parametrize("limit_ms", [2, 10])
def test_waits_give_up_and_report(lib, limit_ms):
    el = torch.zeros(2, dtype=torch.int64, device="cuda")
    lib.coli_moe_test_wait_timeout(limit_ms * 1_000_000, el)
    st, flags = lib.coli_moe_get_status()
    assert st == lib._lib.COLI_ERR_DEVICE
    assert flags == lib._lib.COLI_FLAG_TIMEOUT
    e = el.cpu().numpy()
    # each wait lasted at least the limit, and gave up soon after it
    assert np.all(e >= limit_ms * 1_000_000), e
    assert np.all(e < limit_ms * 1_000_000 + 50_000_000), e
    # the status word was cleared by the read
    assert lib.coli_moe_get_status() == (lib._lib.COLI_OK, 0)


def test_hook_refuses_limits_outside_the_kernel_limit(lib):
    for bad in (0, 2_000_000_001):
        with pytest.raises(lib.ColiError):
            lib.coli_moe_test_wait_timeout(bad)


def test_layer_runs_normally_after_a_timeout(lib):
    lib.coli_moe_test_wait_timeout(1_000_000)
    assert lib.coli_moe_get_status()[1] == lib._lib.COLI_FLAG_TIMEOUT
    shape = synth.LayerShape("after_timeout", 256, 256, 16, 2, 1, 4)
    layer = device_layer(shape, seed=9)
    li = synth.LayerInputs(shape, seed=9)
    x = synth.normal_bf16(9, 5, synth.X_IN, (4, 256))
    xd = to_dev_bits(x)
    out = torch.empty_like(xd)
    layer.forward(xd, out, layer.workspace(4))
    assert lib.coli_moe_get_status() == (lib._lib.COLI_OK, 0)
    ref = oracle.moe_layer(oracle_weights(shape, seed=9), x, 16, 2, 1, router_w=li.router_w())
    got, want = oracle.bf16_bits_to_f64(bits(out)), oracle.bf16_bits_to_f64(ref["out"])
    assert np.abs(got - want).max() <= OUT_REL_TOL * np.abs(want).max()
