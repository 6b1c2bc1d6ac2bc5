"""Failure detection on the GPU without a fault: every device-side wait of the
library is bounded; a wait that runs out sets MOE_DEV_WAIT_TIMEOUT in the
status word and the kernel returns, leaving the context usable.  The watchdog
self-test entry point runs the library's own bounded waits (the FFN's
cluster-scope and CTA-scope mbarrier waits) on a barrier that nothing arrives
at, with a 20 ms limit."""
import time

import pytest
import torch

from combine_moe_route_12_b200 import moe
from combine_moe_route_12_b200.workload import MoEWorkload, make_inputs
from moe_testlib import assert_routing_equal, oracle_routing, run_gpu_steps, to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("which", [0, 1])
def test_wait_that_runs_out_is_reported_and_the_context_survives(which):
    wl = MoEWorkload("watchdog", T=64, H=128, E=8, k=2, I=64, dtype="bf16", ep=2)
    cfg = moe.config_from_workload(wl)
    ws = moe.alloc_workspace(moe.workspace_bytes(cfg))
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    moe.moe_watchdog_selftest(cfg, which, 20000, ws)
    flags = moe.moe_device_status(ws)
    dt = time.perf_counter() - t0
    assert flags == moe.MOE_DEV_WAIT_TIMEOUT
    assert 0.015 < dt < 1.5, dt          # the wait ran its limit out, then returned
    assert moe.moe_device_status(ws) == 0  # read and cleared
    # the same context still computes the layer exactly
    inp = make_inputs(wl, "cpu", seed=4)
    g = run_gpu_steps(wl, to_device(inp))
    assert g["status"] == 0
    assert_routing_equal(g, oracle_routing(wl, inp), wl)


def test_selftest_rejects_bad_arguments():
    wl = MoEWorkload("watchdog", T=64, H=128, E=8, k=2, I=64, dtype="bf16", ep=2)
    cfg = moe.config_from_workload(wl)
    ws = moe.alloc_workspace(moe.workspace_bytes(cfg))
    for which, limit in ((2, 1000), (0, 0), (1, 3000000)):
        with pytest.raises(moe.MoEError):
            moe.moe_watchdog_selftest(cfg, which, limit, ws)
