"""Failure detection on the GPU without a fault: the library's bounded waits
give up on a condition that nothing satisfies, record MOE_DEV_TIMEOUT in the
per-device status word and return; the context stays usable afterwards."""
import time

import pytest
import torch

import combine_moe_route_14_b200 as moe
from combine_moe_route_14_b200 import inputs as I

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TIMEOUT_BIT = 0x2


# 0: readiness counts, 1: ring mbarrier, 2: combine flag bit, 3: queue mbarrier (cluster scope)
@pytest.mark.parametrize("which", [0, 1, 2, 3])
def test_bounded_wait_times_out_and_reports(cuda_lib, which):
    moe.moe_device_status(clear=True)
    counter = torch.zeros(1, dtype=torch.int32, device=DEV) if which in (0, 2) else None
    t0 = time.perf_counter()
    moe.moe_selftest_bounded_wait(which, 50_000, counter)  # 50 ms
    bits = moe.moe_device_status(clear=True)  # synchronises
    dt = time.perf_counter() - t0
    assert bits & TIMEOUT_BIT
    assert 0.04 <= dt < 5.0  # the wait ran to its limit and then returned
    # the context is still usable: a full layer runs and leaves no status bits
    cfg = I.workload("tiny")
    inp = I.make_layer_inputs(cfg, 0, device=DEV)
    layer = moe.MoeLayer(inp["W1"], inp["W2"], cfg.k, cfg.score, cfg.renormalize)
    Y = layer(inp["X"].to(DEV), logits=inp["logits"].to(DEV))
    assert moe.moe_device_status(clear=True) == 0
    assert torch.isfinite(Y.float()).all()


def test_selftest_rejects_bad_arguments(cuda_lib):
    with pytest.raises(moe.MoeError):
        moe.moe_selftest_bounded_wait(4, 1000)
    with pytest.raises(moe.MoeError):
        moe.moe_selftest_bounded_wait(1, 0)
