"""Helpers shared by the GPU parity tests: run every ABI step of the CUDA path
on one set of inputs, run the CPU oracle on the same inputs, and compare.

Tolerances (from the layer's stated contract): indices, drop sets, layouts,
split counts, routing weights and permuted rows bit-exact; floating outputs
within max-abs 1e-4 (fp32) or max|a-b| / max|ref| <= 2e-2 (bf16, fp32
accumulate).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from combine_moe_route_12_b200 import moe
from combine_moe_route_12_b200.workload import MoEInputs, MoEWorkload

F32_ABS_TOL = 1e-4
BF16_REL_TOL = 2e-2


def storage_np(t: torch.Tensor) -> np.ndarray:
    """CPU numpy copy in oracle storage form (float32, or uint16 bf16 bits)."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16).copy()
    return t.numpy().copy()


def storage_f64(a: np.ndarray) -> np.ndarray:
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def assert_float_close(got: np.ndarray, ref: np.ndarray, dtype: str, what: str) -> float:
    g = storage_f64(got) if got.dtype == np.uint16 else got.astype(np.float64)
    r = storage_f64(ref) if ref.dtype == np.uint16 else ref.astype(np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite values"
    if g.size == 0:
        return 0.0
    err = float(np.max(np.abs(g - r)))
    if dtype == "f32":
        assert err <= F32_ABS_TOL, f"{what}: max abs err {err:.3e} > {F32_ABS_TOL}"
        return err
    scale = float(np.max(np.abs(r)))
    rel = err / scale if scale > 0 else err
    assert rel <= BF16_REL_TOL, f"{what}: max err {err:.3e} / max|ref| {scale:.3e} = {rel:.3e}"
    return rel


def to_device(inp: MoEInputs, device="cuda") -> MoEInputs:
    mv = lambda t: None if t is None else t.to(device)
    return MoEInputs(logits=mv(inp.logits), bias=mv(inp.bias), x=mv(inp.x), w13=mv(inp.w13),
                     w2=mv(inp.w2), w13s=mv(inp.w13s), w2s=mv(inp.w2s))


def run_gpu_steps(wl: MoEWorkload, inp: MoEInputs, keep_rows: bool = True) -> dict:
    """Runs the six ABI steps chunk by chunk on the current CUDA stream."""
    cfg = moe.config_from_workload(wl)
    dev = inp.logits.device
    T, E, k, H, I, ep = wl.T, wl.E, wl.k, wl.H, wl.I, wl.ep
    ws = moe.alloc_workspace(moe.workspace_bytes(cfg), dev)
    topk_idx = torch.full((T, k), -7, dtype=torch.int32, device=dev)
    topk_w = torch.full((T, k), -7.0, dtype=torch.float32, device=dev)
    counts = torch.full((E,), -7, dtype=torch.int32, device=dev)
    keep = torch.full((T, k), 7, dtype=torch.uint8, device=dev)
    kept = torch.full((E,), -7, dtype=torch.int32, device=dev)
    moe.moe_route_topk(cfg, inp.logits, inp.bias, topk_idx, topk_w, counts, ws)
    moe.moe_capacity_clip(cfg, topk_idx, topk_w, counts, keep, kept, ws)
    out = torch.full((T, H), float("nan"), dtype=wl.torch_dtype, device=dev)
    red = torch.zeros((T, H), dtype=torch.float32, device=dev) if wl.reduce_dense else None
    tc = T // wl.n_chunks
    nmax = moe.max_recv_rows(cfg, tc)
    chunks = []
    for c in range(wl.n_chunks):
        tb = c * tc
        eoff = torch.full((E + 1,), -7, dtype=torch.int32, device=dev)
        roff = torch.full((ep + 1,), -7, dtype=torch.int32, device=dev)
        rt = torch.full((max(nmax, 1),), -7, dtype=torch.int32, device=dev)
        rs = torch.full((max(nmax, 1),), -7, dtype=torch.int32, device=dev)
        pos = torch.full((tc, k), -7, dtype=torch.int32, device=dev)
        spl = torch.full((ep, ep), -7, dtype=torch.int32, device=dev)
        host = torch.full((E + 1 + ep * ep,), -7, dtype=torch.int32).pin_memory()
        moe.moe_dispatch_layout(cfg, tb, tc, topk_idx, keep, eoff, roff, rt, rs, pos, spl, host, ws)
        xr = torch.empty((max(nmax, 1), H), dtype=wl.torch_dtype, device=dev)
        moe.moe_permute(cfg, inp.x, pos, tb, tc, xr)
        h = torch.empty((max(nmax, 1), I), dtype=wl.torch_dtype, device=dev)
        y = None if wl.reduce_dense else torch.empty((max(nmax, 1), H), dtype=wl.torch_dtype, device=dev)
        moe.moe_grouped_swiglu_ffn(cfg, nmax, xr, eoff, inp.w13, inp.w2, h, y, rt, rs, topk_w, red, ws)
        ys = None
        if wl.shared_I > 0:
            hs = torch.empty((tc, wl.shared_I), dtype=wl.torch_dtype, device=dev)
            ys = torch.empty((tc, H), dtype=wl.torch_dtype, device=dev)
            moe.moe_shared_expert_ffn(cfg, tb, tc, inp.x, inp.w13s, inp.w2s, hs, ys, ws)
        if wl.reduce_dense:
            moe.moe_reduce_finalize(cfg, red, tb, tc, out, y_shared=ys)
        else:
            moe.moe_combine(cfg, y, pos, topk_w, tb, tc, out, y_shared=ys)
        torch.cuda.synchronize()
        n = int(eoff[E].item())
        ch = dict(N=n, expert_offsets=eoff.cpu().numpy(), rank_offsets=roff.cpu().numpy(),
                  recv_token=rt[:n].cpu().numpy(), recv_slot=rs[:n].cpu().numpy(),
                  pos=pos.cpu().numpy(), send_splits=spl.cpu().numpy(), host=host.numpy().copy())
        if keep_rows:
            ch.update(xr=storage_np(xr[:n]), h=storage_np(h[:n]),
                      y=None if y is None else storage_np(y[:n]),
                      ys=None if ys is None else storage_np(ys))
        else:
            ch.update(xr_dev=xr, h_dev=h, y_dev=y, ys_dev=ys)
        chunks.append(ch)
    status = moe.moe_device_status(ws)
    torch.cuda.synchronize()
    return dict(topk_idx=topk_idx.cpu().numpy(), topk_w=topk_w.cpu().numpy(),
                counts=counts.cpu().numpy(), keep=keep.cpu().numpy(), kept_counts=kept.cpu().numpy(),
                chunks=chunks, out=out, status=status)


def oracle_routing(wl: MoEWorkload, inp: MoEInputs) -> dict:
    logits = inp.logits.detach().cpu().numpy()
    bias = None if inp.bias is None else inp.bias.detach().cpu().numpy()
    idx, w, counts, st = oracle.route_topk(logits, bias, wl.k, wl.n_group, wl.topk_group,
                                           wl.group_score, wl.bias_select_only)
    assert st == oracle.ORC_OK
    keep, kept = oracle.capacity_clip(idx, w, wl.E, wl.capacity)
    tc = wl.T // wl.n_chunks
    lays = [oracle.dispatch_layout(idx, keep, wl.E, wl.ep, c * tc, tc) for c in range(wl.n_chunks)]
    return dict(topk_idx=idx, topk_w=w, counts=counts, keep=keep, kept_counts=kept, layouts=lays)


def assert_routing_equal(g: dict, o: dict, wl: MoEWorkload) -> None:
    np.testing.assert_array_equal(g["topk_idx"], o["topk_idx"])
    np.testing.assert_array_equal(g["topk_w"].view(np.uint32), o["topk_w"].view(np.uint32))
    np.testing.assert_array_equal(g["counts"], o["counts"])
    np.testing.assert_array_equal(g["keep"], o["keep"])
    np.testing.assert_array_equal(g["kept_counts"], o["kept_counts"])
    for gc, oc in zip(g["chunks"], o["layouts"]):
        assert gc["N"] == oc["N"]
        for key in ("expert_offsets", "rank_offsets", "recv_token", "recv_slot", "pos", "send_splits"):
            np.testing.assert_array_equal(gc[key], oc[key], err_msg=key)
        np.testing.assert_array_equal(gc["host"][:wl.E + 1], oc["expert_offsets"])
        np.testing.assert_array_equal(gc["host"][wl.E + 1:].reshape(wl.ep, wl.ep), oc["send_splits"])
