"""The allocation-free dispatch layout (moe_dispatch_layout_noalloc) against the
workspace entry point (moe_dispatch_layout), through the C ABI.

It serves callers that cannot allocate device memory (a stream being captured
by another framework, a fixed memory pool, latency-critical loops); its
scratch is a library-owned device array that every call reuses, so two calls
in a row are checked: the second must not see the first one's leftovers.
Layouts are integer results, so the bar is bit-exact equality.  This file is
collected last on purpose.
"""
import numpy as np
import pytest
import torch

from combine_moe_route_12_b200 import moe
from combine_moe_route_12_b200.workload import MoEWorkload, make_inputs

pytestmark = pytest.mark.gpu


def _layout(fn, cfg, wl, tb, tc, idx, keep, **kw):
    nmax = moe.max_recv_rows(cfg, tc)
    d = dict(
        eoff=torch.full((wl.E + 1,), -3, dtype=torch.int32, device="cuda"),
        roff=torch.full((wl.ep + 1,), -3, dtype=torch.int32, device="cuda"),
        rt=torch.full((max(nmax, 1),), -3, dtype=torch.int32, device="cuda"),
        rs=torch.full((max(nmax, 1),), -3, dtype=torch.int32, device="cuda"),
        pos=torch.full((tc, wl.k), -3, dtype=torch.int32, device="cuda"),
        spl=torch.full((wl.ep, wl.ep), -3, dtype=torch.int32, device="cuda"),
        host=torch.full((wl.E + 1 + wl.ep * wl.ep,), -3, dtype=torch.int32).pin_memory(),
    )
    fn(cfg, tb, tc, idx, keep, d["eoff"], d["roff"], d["rt"], d["rs"], d["pos"], d["spl"], d["host"], **kw)
    torch.cuda.synchronize()
    n = int(d["eoff"][wl.E].item())
    return {k: (v[:n] if k in ("rt", "rs") else v).cpu().numpy() for k, v in d.items()}, n


# (workload, token ranges): two calls in a row on different ranges (the second
# reuses the array the first one left behind), then the first range again; the
# second workload fills the array to its edge - 64 tiles of 256 tokens times
# 1024 experts of per-tile counts - and takes the scatter's shared-memory
# opt-in beyond 48 KiB
CASES = [
    (MoEWorkload("noalloc", T=2048, H=128, E=64, k=6, I=128, dtype="bf16", ep=4,
                 capacity=150, skew_bias=True), ((0, 2048), (512, 1024), (0, 2048))),
    (MoEWorkload("noalloc_edge", T=16384, H=128, E=1024, k=8, I=128, dtype="bf16", ep=8),
     ((0, 16384), (8192, 4096), (0, 16384))),
]


@pytest.mark.parametrize("wl,ranges", CASES, ids=[c[0].name for c in CASES])
def test_noalloc_layout_equals_workspace_layout_twice(wl, ranges):
    cfg = moe.config_from_workload(wl)
    inp = make_inputs(wl, "cuda", seed=5, weights=False)
    ws = moe.alloc_workspace(moe.workspace_bytes(cfg))
    idx = torch.empty(wl.T, wl.k, dtype=torch.int32, device="cuda")
    w = torch.empty(wl.T, wl.k, device="cuda")
    counts = torch.empty(wl.E, dtype=torch.int32, device="cuda")
    keep = torch.empty(wl.T, wl.k, dtype=torch.uint8, device="cuda")
    kept = torch.empty(wl.E, dtype=torch.int32, device="cuda")
    moe.moe_route_topk(cfg, inp.logits, inp.bias, idx, w, counts, ws)
    moe.moe_capacity_clip(cfg, idx, w, counts, keep, kept, ws)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for tb, tc in ranges:
        ref, n_ref = _layout(lambda *a: moe.moe_dispatch_layout(*a, ws), cfg, wl, tb, tc, idx, keep)
        got, n_got = _layout(moe.moe_dispatch_layout_noalloc, cfg, wl, tb, tc, idx, keep,
                             status=status)
        assert n_got == n_ref > 0
        for key in ref:
            np.testing.assert_array_equal(got[key], ref[key], err_msg=f"{key} tb={tb} tc={tc}")
    assert int(status.item()) == 0
    assert moe.moe_device_status(ws) == 0


def test_noalloc_layout_rejects_oversized_calls():
    wl = MoEWorkload("noalloc_big", T=32768, H=128, E=8, k=2, I=128, dtype="bf16", ep=2)
    cfg = moe.config_from_workload(wl)
    z = torch.zeros(16, dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_dispatch_layout_noalloc(cfg, 0, 32768, z, z, z, z, z, z, z, z, None)
    assert ei.value.status == moe.MOE_ERR_UNSUPPORTED
    assert "16384" in str(ei.value)
