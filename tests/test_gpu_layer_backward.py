"""The layer's backward on the GPU (moe_layer_backward) with the dispatch outputs
saved by the forward (moe_forward_chunked_save) or recomputed, against each
other (the same bits) and against the oracle's layer backward (fp64, h and y
unrounded; pinned by central finite differences of the forward oracle).

axolotl ExpertParallelArgs, expert_parallel_save_dispatch: under activation
checkpointing the dispatch / combine outputs are held for the backward or the
exchanges are issued again; the routing top-k and the split counts are kept
either way.  Cases: fp32 and bf16, two chunks with a binding capacity, a
shared expert, grouped top-k with a bias that steers the selection only.
Bar: fp32 max-abs 1e-4, bf16 max|a-b| / max|ref| <= 2e-2 per tensor (per
expert for the weight gradients).
"""
import numpy as np
import pytest
import torch

import oracle
from combine_moe_route_12_b200 import moe
from combine_moe_route_12_b200.workload import MoEWorkload, make_inputs

from moe_testlib import assert_float_close, storage_f64, storage_np

pytestmark = pytest.mark.gpu

W = MoEWorkload
CASES = {
    "f32_chunked_cap": W("f32_chunked_cap", T=256, H=128, E=8, k=2, I=128, dtype="f32", ep=2,
                         capacity=48, n_chunks=2),
    "bf16_chunked_cap": W("bf16_chunked_cap", T=512, H=256, E=16, k=4, I=128, dtype="bf16", ep=4,
                          capacity=100, n_chunks=2, skew_bias=True),
    "bf16_shared": W("bf16_shared", T=256, H=128, E=8, k=2, I=128, dtype="bf16", ep=2, n_chunks=2,
                     shared_I=128),
    "bf16_grouped_selbias": W("bf16_grouped_selbias", T=256, H=128, E=16, k=4, I=64, dtype="bf16",
                              ep=2, n_group=4, topk_group=2, group_score=1, bias_select_only=True,
                              balance_bias=True),
}


def _gpu_backward(wl, inp, dout, saved):
    cfg = moe.config_from_workload(wl)
    dev = "cuda"
    T, H, E, k, I = wl.T, wl.H, wl.E, wl.k, wl.I
    dt = wl.torch_dtype
    nmax = moe.max_recv_rows(cfg, T // wl.n_chunks)
    fws = moe.alloc_workspace(moe.forward_workspace_bytes(cfg), dev)
    idx = torch.empty(T, k, dtype=torch.int32, device=dev)
    w = torch.empty(T, k, dtype=torch.float32, device=dev)
    keep = torch.empty(T, k, dtype=torch.uint8, device=dev)
    out = torch.empty(T, H, dtype=dt, device=dev)
    xr_s = torch.zeros(wl.n_chunks, max(nmax, 1), H, dtype=dt, device=dev)
    y_s = torch.zeros(wl.n_chunks, max(nmax, 1), H, dtype=dt, device=dev)
    s = torch.cuda.current_stream()
    moe.moe_forward_chunked_save(cfg, inp.logits, inp.bias, inp.x, inp.w13, inp.w2, out, idx, w, keep,
                                 None, xr_s, y_s, fws, s, s, inp.w13s, inp.w2s)
    # the saving forward gives the plain forward's bits
    out_plain = torch.empty_like(out)
    moe.moe_forward_chunked(cfg, inp.logits, inp.bias, inp.x, inp.w13, inp.w2, out_plain, idx, w, keep,
                            None, fws, s, s, inp.w13s, inp.w2s)
    assert torch.equal(out, out_plain)
    bws = moe.alloc_workspace(moe.backward_workspace_bytes(cfg), dev)
    res = {}
    for mode in ("save", "recompute"):
        g = dict(dx=torch.full((T, H), float("nan"), dtype=dt, device=dev),
                 dlogits=torch.full((T, E), float("nan"), device=dev),
                 dbias=torch.full((E,), float("nan"), device=dev),
                 dw13=torch.full((E, 2 * I, H), float("nan"), device=dev),
                 dw2=torch.full((E, H, I), float("nan"), device=dev))
        if wl.shared_I > 0:
            g["dw13s"] = torch.full((2 * wl.shared_I, H), float("nan"), device=dev)
            g["dw2s"] = torch.full((H, wl.shared_I), float("nan"), device=dev)
        moe.moe_layer_backward(cfg, inp.x, dout, inp.w13, inp.w2, idx, w, keep, g["dx"], g["dlogits"],
                               g["dbias"], g["dw13"], g["dw2"], bws,
                               xr_saved=xr_s if mode == "save" else None,
                               y_saved=y_s if mode == "save" else None,
                               w13_shared=inp.w13s, w2_shared=inp.w2s,
                               dw13_shared=g.get("dw13s"), dw2_shared=g.get("dw2s"))
        torch.cuda.synchronize()
        assert moe.moe_device_status(bws) == 0
        res[mode] = g
    assert moe.moe_device_status(fws) == 0
    return res, idx.cpu().numpy(), w.cpu().numpy(), keep.cpu().numpy()


@pytest.mark.parametrize("name", sorted(CASES))
def test_layer_backward_save_equals_recompute_and_oracle(name):
    wl = CASES[name]
    inp = make_inputs(wl, "cuda", seed=7)
    gen = torch.Generator(device="cuda").manual_seed(99)
    dout = torch.randn(wl.T, wl.H, generator=gen, device="cuda").to(wl.torch_dtype)
    res, idx, w, keep = _gpu_backward(wl, inp, dout, True)
    a, b = res["save"], res["recompute"]
    for key in a:
        assert torch.equal(a[key], b[key]), f"save and recompute differ in {key}"

    x = storage_np(inp.x)
    ref = oracle.moe_layer_backward(
        inp.logits.cpu().numpy(), None if inp.bias is None else inp.bias.cpu().numpy(), x,
        storage_np(inp.w13), storage_np(inp.w2), wl.k, wl.ep, storage_f64(storage_np(dout)),
        wl.capacity, wl.n_chunks, wl.n_group, wl.topk_group, wl.group_score, wl.bias_select_only,
        None if inp.w13s is None else storage_np(inp.w13s),
        None if inp.w2s is None else storage_np(inp.w2s))
    # the saved routing is the oracle's
    np.testing.assert_array_equal(idx, ref["topk_idx"])
    np.testing.assert_array_equal(w.view(np.uint32), ref["topk_w"].view(np.uint32))
    np.testing.assert_array_equal(keep, ref["keep"])
    dt = wl.dtype
    assert_float_close(storage_np(a["dx"]), ref["dx"], dt, "dx")
    assert_float_close(a["dlogits"].cpu().numpy(), ref["dlogits"], dt, "dlogits")
    if inp.bias is not None:
        db = a["dbias"].cpu().numpy()
        if wl.bias_select_only:
            assert (db == 0).all()
        else:
            assert_float_close(db, ref["dbias"], dt, "dbias")
    dw13 = a["dw13"].cpu().numpy().astype(np.float64)
    dw2 = a["dw2"].cpu().numpy().astype(np.float64)
    for e in range(wl.E):
        if not np.any(ref["dW2"][e]):
            assert (dw13[e] == 0).all() and (dw2[e] == 0).all(), f"expert {e} without rows"
            continue
        assert_float_close(dw13[e], ref["dW13"][e], dt, f"dW13[{e}]")
        assert_float_close(dw2[e], ref["dW2"][e], dt, f"dW2[{e}]")
    if wl.shared_I > 0:
        assert_float_close(a["dw13s"].cpu().numpy().astype(np.float64), ref["dW13_shared"], dt, "dW13_shared")
        assert_float_close(a["dw2s"].cpu().numpy().astype(np.float64), ref["dW2_shared"], dt, "dW2_shared")
