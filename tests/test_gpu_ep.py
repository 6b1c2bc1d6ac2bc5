"""The expert-parallel exchange on the GPU (`combine_moe_route_12_b200.ep`).

- `moe_ep_regroup` against numpy: source-major cells to expert-major and back,
  with empty cells, whole experts without rows, one source and eight; the local
  expert offsets it writes; a count table that does not add up to the rows sets
  the status bit and touches nothing past the rows.
- EP ranks emulated in one process: each rank's phases (dispatch, experts,
  combine) run the library's kernels on its own tokens and experts, and the test
  moves the rows between the ranks as the two all-to-alls would (no rank waits on
  another: the ranks run one after the other).  The combined output of every rank
  equals, bit for bit, the single-GPU layer over the whole batch: each row's
  expert output does not depend on which rows share its tile, and the combine
  sums a token's rows in the same slot order.  One case routes every token to the
  first rank's experts, so the other ranks receive no rows at all.
- `EPRank.forward` over a one-rank NCCL group (the collectives with one rank) equals
  the single-GPU layer bitwise.
"""
import os
import socket

import numpy as np
import pytest
import torch

from combine_moe_route_12_b200 import ep, moe
from combine_moe_route_12_b200.workload import MoEWorkload, make_inputs

pytestmark = pytest.mark.gpu


def _regroup_ref(counts, rows):
    """numpy: the expert-major order of source-major rows (the destination index
    of each source-major row)."""
    n_src, n_exp = counts.shape
    src_start = np.concatenate([[0], np.cumsum(counts.reshape(-1))])[:-1].reshape(n_src, n_exp)
    dst = np.empty(rows, np.int64)
    q = 0
    for e in range(n_exp):
        for s in range(n_src):
            for i in range(counts[s, e]):
                dst[src_start[s, e] + i] = q
                q += 1
    exp_off = np.concatenate([[0], np.cumsum(counts.sum(0))])
    return dst, exp_off


@pytest.mark.parametrize("n_src,n_exp,H,dtype", [(1, 5, 64, "bf16"), (2, 4, 256, "bf16"), (4, 3, 128, "f32"),
                                                  (8, 16, 2048, "bf16")])
def test_regroup_against_numpy(n_src, n_exp, H, dtype):
    g = np.random.default_rng(n_src * 100 + n_exp)
    counts = g.integers(0, 7, (n_src, n_exp)).astype(np.int32)
    counts[:, n_exp // 2] = 0          # an expert no source sends rows to
    counts[n_src - 1, 0] = 0
    rows = int(counts.sum())
    cfg = moe.make_config(8 * n_src, H, n_src * n_exp, 2, 128, n_src, -1, dtype)
    ws = moe.alloc_workspace(moe.workspace_bytes(cfg))
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    x = torch.randn(rows, H, device="cuda").to(tdt)
    out = torch.full((rows, H), float("nan"), device="cuda", dtype=tdt)
    back = torch.full((rows, H), float("nan"), device="cuda", dtype=tdt)
    cnt = torch.from_numpy(counts).cuda()
    offs = torch.full((n_exp + 1,), -5, dtype=torch.int32, device="cuda")
    moe.moe_ep_regroup(cfg, cnt, x, out, rows, 0, ws, offs)
    moe.moe_ep_regroup(cfg, cnt, out, back, rows, 1, ws)
    torch.cuda.synchronize()
    assert moe.moe_device_status(ws) == 0
    dst, exp_off = _regroup_ref(counts, rows)
    want = torch.empty_like(x)
    want[torch.from_numpy(dst).cuda()] = x
    assert torch.equal(out, want)
    assert torch.equal(back, x)
    np.testing.assert_array_equal(offs.cpu().numpy(), exp_off)


def test_regroup_rejects_a_table_that_does_not_add_up():
    n_src, n_exp, H = 2, 4, 64
    counts = np.full((n_src, n_exp), 3, np.int32)
    rows = int(counts.sum()) - 5          # the table claims 5 rows more than given
    cfg = moe.make_config(8 * n_src, H, n_src * n_exp, 2, 128, n_src, -1, "bf16")
    ws = moe.alloc_workspace(moe.workspace_bytes(cfg))
    x = torch.randn(rows + 8, H, device="cuda").to(torch.bfloat16)
    out = torch.zeros(rows + 8, H, device="cuda", dtype=torch.bfloat16)
    moe.moe_ep_regroup(cfg, torch.from_numpy(counts).cuda(), x[:rows], out[:rows], rows, 0, ws)
    torch.cuda.synchronize()
    assert moe.moe_device_status(ws) & moe.MOE_DEV_BAD_INDEX
    assert torch.count_nonzero(out[rows:]) == 0     # nothing written past the rows


def _single_gpu(wl, inp):
    layer = moe.MoELayer(moe.config_from_workload(wl))
    out = torch.empty(wl.T, wl.H, dtype=wl.torch_dtype, device="cuda")
    layer.forward(inp.logits, inp.bias, inp.x, inp.w13, inp.w2, out)
    torch.cuda.synchronize()
    assert moe.moe_device_status(layer.ws) == 0
    return out


def _emulated(wl, inp, ep_size):
    """Every rank's phases in one process; the test plays both all-to-alls."""
    Tl, El = wl.T // ep_size, wl.E // ep_size
    ranks = [ep.EPRank(Tl, wl.H, wl.E, wl.k, wl.I, ep_size, r, wl.dtype) for r in range(ep_size)]
    sl = lambda r: slice(r * Tl, (r + 1) * Tl)
    st = [rk.dispatch(inp.logits[sl(r)], inp.bias, inp.x[sl(r)]) for r, rk in enumerate(ranks)]
    # the count all-to-all: rank d receives row d of every source's table
    recv_counts = [torch.stack([st[s].send_counts[d] for s in range(ep_size)]) for d in range(ep_size)]
    # the row all-to-all: source s's segment for d starts at the sum of its sizes before d
    start = [np.concatenate([[0], np.cumsum(st[s].send_sizes)]) for s in range(ep_size)]
    seg = lambda s, d: st[s].xr[int(start[s][d]):int(start[s][d + 1])]
    ys = []
    for d, rk in enumerate(ranks):
        rows = torch.cat([seg(s, d) for s in range(ep_size)])
        w13 = inp.w13[d * El:(d + 1) * El].contiguous()
        w2 = inp.w2[d * El:(d + 1) * El].contiguous()
        ys.append(rk.experts(rows, recv_counts[d], w13, w2))
    # the reverse all-to-all: rank d's outputs go back, source by source
    outs = []
    for s, rk in enumerate(ranks):
        parts = []
        for d in range(ep_size):
            sizes = [int(st[t].send_sizes[d]) for t in range(ep_size)]
            b = sum(sizes[:s])
            parts.append(ys[d][b:b + sizes[s]])
        y_back = torch.cat(parts)
        assert y_back.shape[0] == st[s].n_rows
        out = torch.empty(Tl, wl.H, dtype=wl.torch_dtype, device="cuda")
        rk.combine(st[s], y_back, out)
        outs.append(out)
    torch.cuda.synchronize()
    for rk in ranks:
        assert rk.status() == 0
    return torch.cat(outs), [int(sum(r.sum(1).tolist())) for r in recv_counts]


W = MoEWorkload
EMU = [
    (W("ep2", T=512, H=256, E=16, k=4, I=256, dtype="bf16", ep=2), 2),
    (W("ep4", T=1024, H=512, E=32, k=8, I=384, dtype="bf16", ep=4), 4),
    (W("ep4_f32", T=256, H=128, E=8, k=2, I=256, dtype="f32", ep=4), 4),
]


@pytest.mark.parametrize("wl,ep_size", EMU, ids=[c[0].name for c in EMU])
def test_emulated_ranks_equal_the_single_gpu_layer(wl, ep_size):
    inp = make_inputs(wl, "cuda", seed=7)
    ref = _single_gpu(wl, inp)
    got, recv_rows = _emulated(wl, inp, ep_size)
    assert sum(recv_rows) == wl.T * wl.k
    assert torch.equal(got, ref)


def test_emulated_ranks_with_every_token_on_the_first_rank():
    wl = W("ep_skew", T=512, H=256, E=16, k=4, I=256, dtype="bf16", ep=4)
    inp = make_inputs(wl, "cuda", seed=9)
    # a bias that puts every top-k slot on experts 0..3 (the first rank's)
    inp.bias = torch.zeros(wl.E, device="cuda")
    inp.bias[:4] = 100.0
    ref = _single_gpu(wl, inp)
    got, recv_rows = _emulated(wl, inp, 4)
    assert recv_rows == [wl.T * wl.k, 0, 0, 0]
    assert torch.equal(got, ref)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_forward_over_a_one_rank_nccl_group():
    import torch.distributed as dist
    from datetime import timedelta
    wl = W("ep1", T=512, H=256, E=16, k=4, I=256, dtype="bf16", ep=1)
    inp = make_inputs(wl, "cuda", seed=3)
    ref = _single_gpu(wl, inp)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=timedelta(seconds=60),
                            device_id=torch.device("cuda:0"))
    try:
        rank = ep.EPRank(wl.T, wl.H, wl.E, wl.k, wl.I, 1, 0, wl.dtype)
        out = torch.empty(wl.T, wl.H, dtype=wl.torch_dtype, device="cuda")
        rank.forward(inp.logits, inp.bias, inp.x, inp.w13, inp.w2, out)
        torch.cuda.synchronize()
        assert rank.status() == 0
    finally:
        dist.destroy_process_group()
    assert torch.equal(out, ref)
