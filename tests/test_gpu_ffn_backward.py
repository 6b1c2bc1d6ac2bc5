"""GPU parity of the expert FFN's backward (moe_grouped_swiglu_ffn_backward)
against the oracle's ffn_backward (fp64, h and y unrounded), element by element.

The backward of the grouped SwiGLU FFN is the gradient of step 5's function
(axolotl ExpertParallelArgs, expert_parallel_save_dispatch: the backward of the
expert GEMMs under activation checkpointing); the oracle's form of it is pinned
by central finite differences of the forward oracle.  Cases span ragged expert
segments (empty, one row, fewer than one 16-row MMA step, more than one
token tile, an exact ring stage, every edge of the tiling's merged last tile),
feature and hidden sizes that are not multiples of a 128-row tile, and the fp32
path.  Tolerances: fp32 max-abs 1e-4, bf16 max|a-b| / max|ref| <= 2e-2 per tensor.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_moe_route_12_b200 import moe

from moe_testlib import assert_float_close, storage_f64, storage_np

pytestmark = pytest.mark.gpu

# (name, dtype, H, I, segment sizes per expert)
CASES = [
    ("f32_tiny", "f32", 128, 256, [37, 0, 64, 1, 90, 12, 200, 108]),
    ("bf16_ragged", "bf16", 256, 256, [0, 1, 15, 17, 128, 129, 300, 40]),
    ("bf16_partial_tiles", "bf16", 192, 192, [5, 300, 0, 77]),
    ("bf16_wide", "bf16", 512, 128, [250, 3, 0, 511, 16, 33, 260, 127, 64, 1, 0, 190, 129, 255, 18, 70]),
    # the token tiling's edges: 256-token tiles, the last one of up to 288 tokens,
    # the shared TMEM part past 224, a second MMA past 256, such tiles back to back
    ("bf16_tile_edges", "bf16", 256, 128, [224, 225, 240, 241, 256, 257, 288, 289, 0, 449, 513, 545, 288, 288, 257]),
]


def _case_tensors(dtype, H, I, sizes, seed):
    g = torch.Generator().manual_seed(seed)
    E = len(sizes)
    N = int(sum(sizes))
    dt = torch.float32 if dtype == "f32" else torch.bfloat16
    std = 1.0 / np.sqrt(H)
    xr = torch.randn(max(N, 1), H, generator=g).to(dt)
    dy = (0.5 * torch.randn(max(N, 1), H, generator=g)).to(dt)
    w13 = (torch.randn(E, 2 * I, H, generator=g) * std).to(dt)
    w2 = (torch.randn(E, H, I, generator=g) * std).to(dt)
    offs = np.zeros(E + 1, np.int32)
    offs[1:] = np.cumsum(sizes)
    return xr, dy, w13, w2, offs, N


def _run_gpu(dtype, H, I, E, xr, dy, w13, w2, offs, N, accumulate_twice=False):
    cfg = moe.make_config(T=max(N, 1), H=H, E=E, k=1, I=I, ep=1, dtype=dtype)
    dev = "cuda"
    ws = moe.alloc_workspace(moe.workspace_bytes(cfg), dev)
    dt = xr.dtype
    n = max(N, 1)
    xr_d, dy_d = xr.to(dev), dy.to(dev)
    w13_d, w2_d = w13.to(dev), w2.to(dev)
    offs_d = torch.from_numpy(offs).to(dev)
    gu = torch.full((n, 2 * I), float("nan"), dtype=dt, device=dev)
    h = torch.full((n, I), float("nan"), dtype=dt, device=dev)
    dgu = torch.full((n, 2 * I), float("nan"), dtype=dt, device=dev)
    dxr = torch.full((n, H), float("nan"), dtype=dt, device=dev)
    dw13 = torch.full((E, 2 * I, H), float("nan"), dtype=torch.float32, device=dev)
    dw2 = torch.full((E, H, I), float("nan"), dtype=torch.float32, device=dev)
    moe.moe_grouped_swiglu_ffn_backward(cfg, n, xr_d, dy_d, offs_d, w13_d, w2_d, gu, h, dgu, dxr,
                                        dw13, dw2, 0, ws)
    first = None
    if accumulate_twice:
        first = (dw13.clone(), dw2.clone())
        moe.moe_grouped_swiglu_ffn_backward(cfg, n, xr_d, dy_d, offs_d, w13_d, w2_d, gu, h, dgu, dxr,
                                            dw13, dw2, 1, ws)
    torch.cuda.synchronize()
    assert moe.moe_device_status(ws) == 0
    return dict(h=h[:N], dgu=dgu[:N], dxr=dxr[:N], dw13=dw13, dw2=dw2, first=first)


@pytest.mark.parametrize("name,dtype,H,I,sizes", CASES, ids=[c[0] for c in CASES])
def test_ffn_backward_against_oracle(name, dtype, H, I, sizes):
    xr, dy, w13, w2, offs, N = _case_tensors(dtype, H, I, sizes, seed=len(name))
    E = len(sizes)
    g = _run_gpu(dtype, H, I, E, xr, dy, w13, w2, offs, N)
    xr_np, w13_np, w2_np = storage_np(xr[:N]), storage_np(w13), storage_np(w2)
    dy64 = storage_f64(storage_np(dy[:N]))
    dxr_ref, dw13_ref, dw2_ref = oracle.ffn_backward(xr_np, offs, w13_np, w2_np, dy64)
    h_ref, _, _ = oracle.ffn(xr_np, offs, w13_np, w2_np)
    assert_float_close(storage_np(g["dxr"]), dxr_ref, dtype, f"{name} dxr")
    assert_float_close(storage_np(g["h"]), h_ref, dtype, f"{name} h")
    # weight gradients: fp32 outputs against the fp64 oracle, per expert with rows
    # (experts without rows must be exactly zero)
    wdt = "f32" if dtype == "f32" else "bf16"
    dw13 = g["dw13"].cpu().numpy().astype(np.float64)
    dw2 = g["dw2"].cpu().numpy().astype(np.float64)
    for e in range(E):
        if sizes[e] == 0:
            assert (dw13[e] == 0).all() and (dw2[e] == 0).all(), f"expert {e} without rows"
            continue
        assert_float_close(dw2[e], dw2_ref[e], wdt, f"{name} dW2[{e}]")
        assert_float_close(dw13[e], dw13_ref[e], wdt, f"{name} dW13[{e}]")


def test_ffn_backward_accumulates_exactly():
    """accumulate = 1 adds the same gradient again: the result is exactly twice
    the first call's (x + x is exact in fp32)."""
    name, dtype, H, I, sizes = CASES[1]
    xr, dy, w13, w2, offs, N = _case_tensors(dtype, H, I, sizes, seed=5)
    g = _run_gpu(dtype, H, I, len(sizes), xr, dy, w13, w2, offs, N, accumulate_twice=True)
    a13, a2 = g["first"]
    assert torch.equal(g["dw13"], 2 * a13)
    assert torch.equal(g["dw2"], 2 * a2)


def test_ffn_backward_without_rows_zeroes_the_weight_gradients():
    cfg = moe.make_config(T=16, H=128, E=4, k=1, I=128, ep=1, dtype="bf16")
    ws = moe.alloc_workspace(moe.workspace_bytes(cfg))
    offs = torch.zeros(5, dtype=torch.int32, device="cuda")
    w13 = torch.zeros(4, 256, 128, dtype=torch.bfloat16, device="cuda")
    w2 = torch.zeros(4, 128, 128, dtype=torch.bfloat16, device="cuda")
    dw13 = torch.full((4, 256, 128), 3.0, device="cuda")
    dw2 = torch.full((4, 128, 128), 3.0, device="cuda")
    moe.moe_grouped_swiglu_ffn_backward(cfg, 0, None, None, offs, w13, w2, None, None, None, None,
                                        dw13, dw2, 0, ws)
    torch.cuda.synchronize()
    assert (dw13 == 0).all() and (dw2 == 0).all()
