"""The grouped FFN at the edges of its token tiling, element by element against
the oracle.

The kernel covers an expert's rows 256 at a time and lets the last tile take up
to 288.  Each TMEM accumulator owns 224 columns; a main MMA of more than 224
tokens extends into a 32-column half of a shared part beside it, and a tile of
more than 256 tokens issues a second MMA (N = 32) into the other half; each
32-column chunk of the accumulators maps to two runs of 16 receive rows.  The
segment sizes here sit on every boundary of that rule: one row, under one 16-row
MMA step, 224 / 225 (into the shared part), 240 / 241, 256 / 257 (the extra MMA),
288 / 289 (the largest single tile, then two), 448 / 449, 512 / 513, 544 / 545
(256 + 288, then three tiles), 736 and an empty expert, several of them back to
back so that tiles writing the shared part follow one another on the same CTA
pair, in both accumulators.  Every row of h and y is compared with the oracle,
for the bf16 store epilogue, the decode form's reduce epilogue and the FP8 path
(row scales on codes).  The backward's modes on the same sizes are in
tests/test_gpu_ffn_backward.py.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_moe_route_12_b200 import moe

from moe_testlib import assert_float_close, storage_np

pytestmark = pytest.mark.gpu

SIZES = [224, 225, 240, 241, 256, 257, 272, 273, 288, 289, 304, 0, 1, 15, 33, 448, 449, 512, 513, 544, 545,
         736, 65, 288, 288, 257, 256, 256, 225]
H, I = 256, 256


def _tensors(seed):
    g = torch.Generator().manual_seed(seed)
    E = len(SIZES)
    N = int(sum(SIZES))
    std = 1.0 / np.sqrt(H)
    xr = torch.randn(N, H, generator=g).to(torch.bfloat16)
    w13 = (torch.randn(E, 2 * I, H, generator=g) * std).to(torch.bfloat16)
    w2 = (torch.randn(E, H, I, generator=g) * std).to(torch.bfloat16)
    offs = np.zeros(E + 1, np.int32)
    offs[1:] = np.cumsum(SIZES)
    return xr, w13, w2, offs, N


def _oracle_bf16(xr, w13, w2, offs):
    return oracle.ffn(storage_np(xr), offs, storage_np(w13), storage_np(w2))


def test_store_epilogue_at_tile_edges():
    xr, w13, w2, offs, N = _tensors(11)
    E = len(SIZES)
    cfg = moe.make_config(T=N, H=H, E=E, k=1, I=I, ep=1, dtype="bf16")
    ws = moe.alloc_workspace(moe.workspace_bytes(cfg))
    h = torch.full((N, I), float("nan"), dtype=torch.bfloat16, device="cuda")
    y = torch.full((N, H), float("nan"), dtype=torch.bfloat16, device="cuda")
    moe.moe_grouped_swiglu_ffn(cfg, N, xr.cuda(), torch.from_numpy(offs).cuda(), w13.cuda(), w2.cuda(), h, y,
                               None, None, None, None, ws)
    torch.cuda.synchronize()
    assert moe.moe_device_status(ws) == 0
    h_ref, y_ref, _ = _oracle_bf16(xr, w13, w2, offs)
    h_np, y_np = storage_np(h), storage_np(y)
    # per expert, so that a wrong row mapping names its segment
    for e in range(E):
        a, b = int(offs[e]), int(offs[e + 1])
        if a == b:
            continue
        assert_float_close(h_np[a:b], h_ref[a:b], "bf16", f"h expert {e} ({b - a} rows)")
        assert_float_close(y_np[a:b], y_ref[a:b], "bf16", f"y expert {e} ({b - a} rows)")


def test_reduce_epilogue_at_tile_edges():
    """Decode form: out_reduce[t] += w[t] * y for each receive row; every row here
    is its own token (a random permutation) with one slot, so each element takes
    one atomic add."""
    xr, w13, w2, offs, N = _tensors(12)
    E = len(SIZES)
    cfg = moe.make_config(T=N, H=H, E=E, k=1, I=I, ep=1, dtype="bf16", reduce_dense=True)
    ws = moe.alloc_workspace(moe.workspace_bytes(cfg))
    rng = np.random.default_rng(5)
    tok = rng.permutation(N).astype(np.int32)
    w = rng.uniform(0.1, 1.0, N).astype(np.float32)
    h = torch.empty((N, I), dtype=torch.bfloat16, device="cuda")
    red = torch.zeros((N, H), dtype=torch.float32, device="cuda")
    moe.moe_grouped_swiglu_ffn(cfg, N, xr.cuda(), torch.from_numpy(offs).cuda(), w13.cuda(), w2.cuda(), h, None,
                               torch.from_numpy(tok).cuda(), torch.zeros(N, dtype=torch.int32, device="cuda"),
                               torch.from_numpy(w).cuda(), red, ws)
    torch.cuda.synchronize()
    assert moe.moe_device_status(ws) == 0
    _, _, y_exact = _oracle_bf16(xr, w13, w2, offs)
    # the weight is read through the token: topk_w[recv_token[p] * k + recv_slot[p]]
    ref = np.zeros((N, H))
    ref[tok] = w[tok][:, None].astype(np.float64) * y_exact
    assert_float_close(red.cpu().numpy(), ref, "bf16", "out_reduce")
    # every token's row written: none left at zero where the reference is not
    assert np.count_nonzero(red.cpu().numpy()) == np.count_nonzero(ref)


def test_fp8_at_tile_edges():
    xr, w13, w2, offs, N = _tensors(13)
    E = len(SIZES)
    xq, xs = oracle.quantize_rows(storage_np(xr))
    w13q, w13s = oracle.quantize_rows(storage_np(w13).reshape(E * 2 * I, H))
    w2q, w2s = oracle.quantize_rows(storage_np(w2).reshape(E * H, I))
    cfg = moe.make_config(T=N, H=H, E=E, k=1, I=I, ep=1, dtype="bf16", ffn_fp8=True)
    ws = moe.alloc_workspace(moe.workspace_bytes(cfg))
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    h = torch.full((N, I), float("nan"), dtype=torch.bfloat16, device="cuda")
    hq = torch.empty((N, I), dtype=torch.uint8, device="cuda")
    hs = torch.empty(N, dtype=torch.uint8, device="cuda")
    y = torch.full((N, H), float("nan"), dtype=torch.bfloat16, device="cuda")
    # GEMM1 reads x's scale through recv_token: the identity here
    ident = torch.arange(N, dtype=torch.int32, device="cuda")
    moe.moe_grouped_swiglu_ffn_fp8(cfg, N, d(xq), d(xs), d(offs), d(w13q).view(E, 2 * I, H), d(w13s),
                                   d(w2q).view(E, H, I), d(w2s), h, hq, hs, y, ident, None, None, None, ws)
    torch.cuda.synchronize()
    assert moe.moe_device_status(ws) == 0
    w13q3, w13s2 = w13q.reshape(E, 2 * I, H), w13s.reshape(E, 2 * I)
    w2q3, w2s2 = w2q.reshape(E, H, I), w2s.reshape(E, H)
    h_np, y_np = storage_np(h), storage_np(y)
    for e in range(E):
        a, b = int(offs[e]), int(offs[e + 1])
        if a == b:
            continue
        h_ref = np.zeros((b - a, I), np.uint16)
        y_ref = np.zeros((b - a, H), np.uint16)
        for p in range(a, b):
            h_ref[p - a], _, _, y_ref[p - a], _ = oracle.ffn_row_fp8(xq[p], xs[p], w13q3[e], w13s2[e], w2q3[e],
                                                                  w2s2[e])
        assert_float_close(h_np[a:b], h_ref, "bf16", f"h expert {e} ({b - a} rows)")
        # y follows h's codes: a code one step off near a rounding boundary moves a
        # whole row a little, so no per-element share check
        assert_float_close(y_np[a:b], y_ref, "bf16", f"y expert {e} ({b - a} rows)", per_element=False)
