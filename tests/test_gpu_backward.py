"""GPU parity of the backward's row passes (the combine's, the routing's and the
permute's backward) against the oracle, on the same seeded inputs: the routing
and layout are the oracle's (uploaded as inputs; the forward tests check the
GPU's are bit-identical), dout, the expert rows y and the receive-row
gradients dxr are synthetic.

Bar: dy in fp32 bit-exact (one rounding of the fp32 product on both sides), in
bf16 within the bf16 bar; dw, dlogits, dbias and dx within max-abs 1e-4 (fp32
storage, fp32 sums against fp64) or the bf16 bar (max|a-b| / max|ref| <= 2e-2).
"""
import numpy as np
import pytest
import torch

import oracle
from combine_moe_route_12_b200 import moe
from combine_moe_route_12_b200.workload import MoEWorkload, make_inputs

from moe_testlib import assert_float_close, oracle_routing, storage_np

pytestmark = pytest.mark.gpu

W = MoEWorkload
CASES = {
    "tiny_f32": W("tiny_f32", T=256, H=128, E=8, k=2, I=256, dtype="f32", ep=2),
    "bf16_capacity": W("bf16_capacity", T=512, H=128, E=16, k=4, I=128, dtype="bf16", ep=4,
                       capacity=64, skew_bias=True),
    "bf16_chunked": W("bf16_chunked", T=512, H=256, E=8, k=2, I=128, dtype="bf16", ep=2, n_chunks=4),
    "bf16_k_all": W("bf16_k_all", T=64, H=64, E=32, k=32, I=64, dtype="bf16", ep=2, capacity=40),
    "bf16_cap0": W("bf16_cap0", T=64, H=128, E=8, k=2, I=128, dtype="bf16", ep=2, capacity=0),
    "bf16_sparse_chunk": W("bf16_sparse_chunk", T=8192, H=256, E=16, k=2, I=64, dtype="bf16",
                           ep=2, capacity=256, skew_bias=True),
    "f32_selbias": W("f32_selbias", T=256, H=128, E=8, k=2, I=128, dtype="f32", ep=2,
                     skew_bias=True, bias_select_only=True),
}


def _store(a: np.ndarray, dtype: str) -> np.ndarray:
    a = a.astype(np.float32)
    if dtype == "f32":
        return a
    return torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def _dev(a: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if a.dtype == np.uint16:
        t = t.view(torch.int16).view(torch.bfloat16)
    return t.cuda()


@pytest.mark.parametrize("name", sorted(CASES))
def test_backward_row_passes_match_oracle(name):
    wl = CASES[name]
    inp = make_inputs(wl, "cpu", seed=3, weights=False)
    orc = oracle_routing(wl, inp)
    cfg = moe.config_from_workload(wl)
    rng = np.random.default_rng(11)
    T, H, k, E = wl.T, wl.H, wl.k, wl.E
    dout = _store(rng.normal(0, 1, (T, H)), wl.dtype)
    dout_d = _dev(dout, wl.dtype)
    w_d = torch.from_numpy(orc["topk_w"]).cuda()
    tc = T // wl.n_chunks
    nmax = moe.max_recv_rows(cfg, tc)
    dw_d = torch.full((T, k), float("nan"), device="cuda")
    dw_ref = np.zeros((T, k))
    dx_d = torch.full((T, H), float("nan"), dtype=wl.torch_dtype, device="cuda")
    dx_ref = np.zeros((T, H), dout.dtype)
    for c, lay in enumerate(orc["layouts"]):
        n = lay["N"]
        y = _store(rng.normal(0, 1, (max(nmax, 1), H)), wl.dtype)
        pos_d = torch.from_numpy(lay["pos"]).cuda()
        # combine backward
        dy_d = torch.full((max(nmax, 1), H), 7.0, dtype=wl.torch_dtype, device="cuda")
        moe.moe_combine_backward(cfg, dout_d, _dev(y, wl.dtype), pos_d, w_d, c * tc, tc, dy_d, dw_d)
        dy_ref, dw_c = oracle.combine_backward(dout, y[:max(n, 1)], lay["pos"], orc["topk_w"], c * tc)
        dw_ref[c * tc:(c + 1) * tc] = dw_c[c * tc:(c + 1) * tc]
        torch.cuda.synchronize()
        got = storage_np(dy_d)
        if n > 0:
            if wl.dtype == "f32":
                np.testing.assert_array_equal(got[:n], dy_ref[:n])
            else:
                assert_float_close(got[:n], dy_ref[:n], "bf16", f"dy chunk {c}")
        assert (got[n:] == storage_np(torch.full((1,), 7.0, dtype=wl.torch_dtype))[0]).all()
        # permute backward (the combine with unit weights)
        dxr = _store(rng.normal(0, 1, (max(nmax, 1), H)), wl.dtype)
        moe.moe_permute_backward(cfg, _dev(dxr, wl.dtype), pos_d, c * tc, tc, dx_d)
        oracle.combine(dxr[:max(n, 1)], lay["pos"], np.ones((T, k), np.float32), T, c * tc, dx_ref)
    torch.cuda.synchronize()
    assert_float_close(dw_d.cpu().numpy(), dw_ref, "f32" if wl.dtype == "f32" else "bf16", "dw")
    assert_float_close(storage_np(dx_d), dx_ref, wl.dtype, "dx")
    # routing backward, fed the oracle's dw (as stored in fp32)
    dw32 = dw_ref.astype(np.float32)
    ws = moe.alloc_workspace(moe.workspace_bytes(cfg))
    dl_d = torch.full((T, E), float("nan"), device="cuda")
    db_d = torch.full((E,), float("nan"), device="cuda")
    moe.moe_route_backward(cfg, torch.from_numpy(orc["topk_idx"]).cuda(), w_d,
                           torch.from_numpy(dw32).cuda(), dl_d, db_d, ws)
    assert moe.moe_device_status(ws) == 0
    dl_ref = oracle.route_backward(orc["topk_idx"], orc["topk_w"], dw32, E)
    dl = dl_d.cpu().numpy()
    assert_float_close(dl, dl_ref, "f32", "dlogits")
    assert (dl[dl_ref == 0] == 0).all()                 # unselected experts: exactly 0
    db = db_d.cpu().numpy()
    if wl.bias_select_only:
        assert not db.any()
    else:
        # fp32 sums of T terms against fp64: bounded by the sum of their magnitudes
        bound = 1e-5 * np.abs(dl_ref).sum(axis=0) + 1e-6
        assert (np.abs(db - dl_ref.sum(axis=0)) <= bound).all()


def test_backward_entry_points_reject_bad_arguments():
    wl = CASES["bf16_capacity"]
    cfg = moe.config_from_workload(wl.with_(reduce_dense=True))
    z = torch.zeros(64, device="cuda")
    with pytest.raises(moe.MoEError):                  # decode form stores no y
        moe.moe_combine_backward(cfg, z, z, z, z, 0, 8, z, z)
    cfg = moe.config_from_workload(wl)
    with pytest.raises(moe.MoEError):                  # a chunk past T
        moe.moe_permute_backward(cfg, z, z, wl.T - 4, 8, z)
