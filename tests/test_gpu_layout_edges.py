"""The dispatch layout against the oracle's layout, bit-exact, at the edges of
its tiling: a chunk smaller than one warp step per tile, k = 1 and k = 32
(thirty-two slots per token: one token per warp step), a chunk of 16384 tokens
(64 tiles of 256), a binding capacity (dropped slots, pos = -1), E = 1024
experts with 64 ranks (a 4096-entry split matrix in shared memory), and chunks
beyond 64 tiles (each tile's column sums run over more than one 32-tile lane stride).
Routing is taken from the GPU's own route + clip, compared here with the
oracle's, so the layout inputs are the oracle's.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_moe_route_12_b200 import moe
from combine_moe_route_12_b200.workload import MoEWorkload, make_inputs

pytestmark = pytest.mark.gpu

W = MoEWorkload
CASES = [
    W("lay_tiny", T=12, H=128, E=8, k=2, I=128, dtype="bf16", ep=4),
    W("lay_k1", T=4096, H=128, E=64, k=1, I=128, dtype="bf16", ep=2),
    W("lay_k32", T=1024, H=128, E=64, k=32, I=128, dtype="bf16", ep=8, capacity=300, skew_bias=True),
    W("lay_64_tiles", T=16384, H=128, E=128, k=8, I=128, dtype="bf16", ep=4),
    W("lay_e1024", T=2048, H=128, E=1024, k=8, I=128, dtype="bf16", ep=64, capacity=10, skew_bias=True),
    W("lay_multi_cta", T=32768, H=128, E=256, k=8, I=128, dtype="bf16", ep=8, capacity=900, skew_bias=True),
    W("lay_multi_k16", T=16384, H=128, E=1024, k=16, I=128, dtype="bf16", ep=8),
]


@pytest.mark.parametrize("wl", CASES, ids=[c.name for c in CASES])
def test_layout_edges_against_oracle(wl):
    cfg = moe.config_from_workload(wl)
    inp = make_inputs(wl, "cuda", seed=11, weights=False)
    ws = moe.alloc_workspace(moe.workspace_bytes(cfg))
    T, E, k, ep = wl.T, wl.E, wl.k, wl.ep
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, device="cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    keep = torch.empty(T, k, dtype=torch.uint8, device="cuda")
    kept = torch.empty(E, dtype=torch.int32, device="cuda")
    moe.moe_route_topk(cfg, inp.logits, inp.bias, idx, w, counts, ws)
    moe.moe_capacity_clip(cfg, idx, w, counts, keep, kept, ws)
    logits = inp.logits.cpu().numpy()
    bias = None if inp.bias is None else inp.bias.cpu().numpy()
    o_idx, o_w, _, st = oracle.route_topk(logits, bias, k)
    assert st == oracle.ORC_OK
    o_keep, _ = oracle.capacity_clip(o_idx, o_w, E, wl.capacity)
    np.testing.assert_array_equal(idx.cpu().numpy(), o_idx)
    np.testing.assert_array_equal(keep.cpu().numpy(), o_keep)
    nmax = max(1, moe.max_recv_rows(cfg, T))
    eoff = torch.full((E + 1,), -3, dtype=torch.int32, device="cuda")
    roff = torch.full((ep + 1,), -3, dtype=torch.int32, device="cuda")
    rt = torch.full((nmax,), -3, dtype=torch.int32, device="cuda")
    rs = torch.full((nmax,), -3, dtype=torch.int32, device="cuda")
    pos = torch.full((T, k), -3, dtype=torch.int32, device="cuda")
    spl = torch.full((ep, ep), -3, dtype=torch.int32, device="cuda")
    host = torch.full((E + 1 + ep * ep,), -3, dtype=torch.int32).pin_memory()
    moe.moe_dispatch_layout(cfg, 0, T, idx, keep, eoff, roff, rt, rs, pos, spl, host, ws)
    torch.cuda.synchronize()
    assert moe.moe_device_status(ws) == 0
    ref = oracle.dispatch_layout(o_idx, o_keep, E, ep, 0, T)
    n = int(eoff[E].item())
    assert n == ref["N"]
    got = dict(expert_offsets=eoff, rank_offsets=roff, recv_token=rt[:n], recv_slot=rs[:n], pos=pos,
               send_splits=spl)
    for key, v in got.items():
        np.testing.assert_array_equal(v.cpu().numpy(), ref[key], err_msg=key)
    np.testing.assert_array_equal(host.numpy()[:E + 1], ref["expert_offsets"])
    np.testing.assert_array_equal(host.numpy()[E + 1:].reshape(ep, ep), ref["send_splits"])
