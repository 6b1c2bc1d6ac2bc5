"""GPU parity of every ABI step against the CPU oracle, element by element, at
sizes the oracle finishes in seconds that still span several tiles and ragged
tails (expert segments that are not multiples of the 128-row tile, an I and
an H that leave partial N tiles).

Bar: routing indices and weights, keep masks, counts, layouts, split counts
(device and host copy) and permuted rows bit-exact; h, y and out within
max-abs 1e-4 (fp32) or max|a-b|/max|ref| <= 2e-2 (bf16 with fp32 accumulate).
"""
import numpy as np
import pytest
import torch

import oracle
from combine_moe_route_12_b200.workload import MoEInputs, MoEWorkload, make_inputs

from moe_testlib import (assert_float_close, assert_routing_equal, oracle_routing,
                         run_gpu_steps, storage_np, to_device)

pytestmark = pytest.mark.gpu

W = MoEWorkload
CASES = {
    # the fp32 workload exactly as specified
    "tiny_f32": W("tiny_f32", T=256, H=128, E=8, k=2, I=256, dtype="f32", ep=2),
    # bf16, ~128 rows per expert: every expert has a ragged last m tile
    "bf16_ragged_m": W("bf16_ragged_m", T=512, H=128, E=8, k=2, I=128, dtype="bf16", ep=2),
    # partial N tiles in both GEMMs (I = 192 = 128 + 64, H = 320 = 256 + 64), K = 5 and 3 blocks
    "bf16_ragged_n": W("bf16_ragged_n", T=384, H=320, E=16, k=4, I=192, dtype="bf16", ep=4),
    # skewed router with a binding capacity
    "bf16_capacity": W("bf16_capacity", T=512, H=128, E=16, k=4, I=128, dtype="bf16", ep=4,
                       capacity=64, skew_bias=True),
    # 256 experts with ~8 rows each, 64 logical ranks of 4 tokens
    "bf16_many_experts": W("bf16_many_experts", T=256, H=128, E=256, k=8, I=64, dtype="bf16", ep=64),
    # chunked dispatch (4 chunks)
    "bf16_chunked": W("bf16_chunked", T=512, H=256, E=8, k=2, I=128, dtype="bf16", ep=2, n_chunks=4),
    # decode: reduce straight into a dense output
    "bf16_decode": W("bf16_decode", T=64, H=256, E=32, k=8, I=128, dtype="bf16", ep=8, capacity=32,
                     reduce_dense=True),
    "f32_decode": W("f32_decode", T=64, H=128, E=8, k=2, I=128, dtype="f32", ep=2, reduce_dense=True),
    # degenerate: k = 1, top-k of all experts, capacity 0, ep = 1
    "bf16_k1": W("bf16_k1", T=128, H=128, E=4, k=1, I=64, dtype="bf16", ep=1),
    "bf16_k_all": W("bf16_k_all", T=64, H=64, E=32, k=32, I=64, dtype="bf16", ep=2, capacity=40),
    "bf16_cap0": W("bf16_cap0", T=64, H=128, E=8, k=2, I=128, dtype="bf16", ep=2, capacity=0),
    # a chunk of 6144 tokens: the dispatch layout takes 128-token tiles (48 of them)
    "bf16_layout_128": W("bf16_layout_128", T=6144, H=64, E=16, k=2, I=64, dtype="bf16", ep=2),
    # 512 experts: the router's 32-lane groups with 16 values per lane
    "bf16_512_experts": W("bf16_512_experts", T=128, H=64, E=512, k=4, I=64, dtype="bf16", ep=4),
    # routing variants: grouped top-k by the best logit of a group
    "bf16_grouped": W("bf16_grouped", T=256, H=128, E=64, k=6, I=64, dtype="bf16", ep=4,
                      n_group=8, topk_group=3, group_score=0),
    # DSV3-like: 8 groups of 32, 4 kept by the sum of their two best, bias in the selection only
    "bf16_grouped_top2_selbias": W("bf16_grouped_top2_selbias", T=256, H=128, E=256, k=8, I=64,
                                   dtype="bf16", ep=8, n_group=8, topk_group=4, group_score=1,
                                   bias_select_only=True, balance_bias=True),
    # grouped with k > 16 (32-lane token groups) and a binding capacity
    "bf16_grouped_k20": W("bf16_grouped_k20", T=128, H=64, E=64, k=20, I=64, dtype="bf16", ep=2,
                          n_group=4, topk_group=2, group_score=1, capacity=40),
    # fp32, skewed bias in the selection only
    "f32_selbias_skew": W("f32_selbias_skew", T=256, H=128, E=8, k=2, I=128, dtype="f32", ep=2,
                          skew_bias=True, bias_select_only=True),
    # a shared expert beside the routed ones (two chunks, and in the decode form)
    "bf16_shared": W("bf16_shared", T=256, H=128, E=16, k=4, I=64, dtype="bf16", ep=2,
                     shared_I=128, n_chunks=2),
    "bf16_shared_decode": W("bf16_shared_decode", T=64, H=256, E=32, k=8, I=128, dtype="bf16",
                            ep=8, capacity=32, reduce_dense=True, shared_I=192),
    "f32_shared": W("f32_shared", T=128, H=128, E=8, k=2, I=128, dtype="f32", ep=2, shared_I=64),
    # a large chunk (8192 tokens) with most slots dropped: the warp-per-token permute
    # and combine (tokens with no kept row at all among them)
    "bf16_sparse_chunk": W("bf16_sparse_chunk", T=8192, H=256, E=16, k=2, I=64, dtype="bf16",
                           ep=2, capacity=256, skew_bias=True),
}


def _oracle_ffn_and_out(wl, inp, orc):
    x = storage_np(inp.x)
    w13 = storage_np(inp.w13)
    w2 = storage_np(inp.w2)
    res = []
    out = np.zeros((wl.T, wl.H), x.dtype)
    tc = wl.T // wl.n_chunks
    for c, lay in enumerate(orc["layouts"]):
        xr = oracle.permute(x, lay["recv_token"])
        h, y, ye = oracle.ffn(xr, lay["expert_offsets"], w13, w2)
        ys = None
        if wl.shared_I > 0:
            _, ys, _ = oracle.shared_expert(x[c * tc:(c + 1) * tc], storage_np(inp.w13s),
                                            storage_np(inp.w2s))
        if wl.reduce_dense:
            oracle.combine_exact(ye, lay["pos"], orc["topk_w"], wl.T, x.dtype, c * tc, out, y_shared=ys)
        else:
            oracle.combine(y, lay["pos"], orc["topk_w"], wl.T, c * tc, out, y_shared=ys)
        res.append(dict(xr=xr, h=h, y=y, ys=ys))
    return res, out


@pytest.mark.parametrize("name", sorted(CASES))
def test_layer_steps_match_oracle(name):
    wl = CASES[name]
    inp = make_inputs(wl, "cpu", seed=1)
    dinp = to_device(inp)
    g = run_gpu_steps(wl, dinp)
    assert g["status"] == 0
    orc = oracle_routing(wl, inp)
    assert_routing_equal(g, orc, wl)
    rows, out = _oracle_ffn_and_out(wl, inp, orc)
    for gc, oc in zip(g["chunks"], rows):
        np.testing.assert_array_equal(gc["xr"], oc["xr"])            # permute is a bitwise copy
        assert_float_close(gc["h"], oc["h"], wl.dtype, "h")
        if not wl.reduce_dense:
            assert_float_close(gc["y"], oc["y"], wl.dtype, "y")
        if oc["ys"] is not None:
            assert_float_close(gc["ys"], oc["ys"], wl.dtype, "y_shared")
    assert_float_close(storage_np(g["out"]), out, wl.dtype, "out")
    if wl.capacity == 0:
        assert (storage_np(g["out"]) == 0).all()


def _forward(wl, dinp, n_chunks, same_stream=False):
    from combine_moe_route_12_b200 import moe
    wl = wl.with_(n_chunks=n_chunks)
    layer = moe.MoELayer(moe.config_from_workload(wl))
    out = torch.full((wl.T, wl.H), float("nan"), dtype=wl.torch_dtype, device="cuda")
    s = torch.cuda.current_stream()
    if same_stream:
        moe.moe_forward_chunked(layer.cfg, dinp.logits, dinp.bias, dinp.x, dinp.w13, dinp.w2, out,
                                layer.topk_idx, layer.topk_w, layer.keep, layer.splits_host,
                                layer.ws, s, s, dinp.w13s, dinp.w2s)
    else:
        layer.forward(dinp.logits, dinp.bias, dinp.x, dinp.w13, dinp.w2, out,
                      w13_shared=dinp.w13s, w2_shared=dinp.w2s)
    torch.cuda.synchronize()
    assert moe.moe_device_status(layer.ws) == 0
    return out, layer


@pytest.mark.parametrize("name", ["bf16_ragged_m", "bf16_capacity", "bf16_chunked", "tiny_f32",
                                  "bf16_decode", "bf16_shared", "bf16_shared_decode",
                                  "bf16_grouped_top2_selbias", "bf16_sparse_chunk"])
def test_forward_chunked_matches_steps_and_oracle(name):
    wl = CASES[name]
    inp = make_inputs(wl, "cpu", seed=2)
    dinp = to_device(inp)
    out_c, layer = _forward(wl, dinp, wl.n_chunks)
    orc = oracle_routing(wl, inp)
    np.testing.assert_array_equal(layer.topk_idx.cpu().numpy(), orc["topk_idx"])
    np.testing.assert_array_equal(layer.keep.cpu().numpy(), orc["keep"])
    for c, lay in enumerate(orc["layouts"]):
        eoff, spl = layer.splits(c)
        np.testing.assert_array_equal(eoff.numpy(), lay["expert_offsets"])
        np.testing.assert_array_equal(spl.numpy(), lay["send_splits"])
    _, out = _oracle_ffn_and_out(wl, inp, orc)
    assert_float_close(storage_np(out_c), out, wl.dtype, "out")
    if not wl.reduce_dense:
        # the step-by-step path runs the same kernels: identical bits
        g = run_gpu_steps(wl, dinp)
        np.testing.assert_array_equal(storage_np(out_c), storage_np(g["out"]))
        # chunking changes only the overlap, not the result (rows are independent,
        # fixed K order, slot-ordered combine)
        out_1, _ = _forward(wl, dinp, 1)
        np.testing.assert_array_equal(storage_np(out_c), storage_np(out_1))
        out_s, _ = _forward(wl, dinp, wl.n_chunks, same_stream=True)
        np.testing.assert_array_equal(storage_np(out_c), storage_np(out_s))


@pytest.mark.parametrize("name", ["bf16_chunked", "tiny_f32", "bf16_decode", "bf16_shared",
                                  "bf16_grouped_top2_selbias", "f32_shared"])
def test_forward_host_equals_device_forward(name):
    """The host-buffer entry point stages the activations in its workspace and
    copies the output back chunk by chunk; its result is the device forward's,
    bit for bit (the decode form: within tolerance), also for two calls
    enqueued back to back on one workspace."""
    from combine_moe_route_12_b200 import moe
    wl = CASES[name]
    inps = [make_inputs(wl, "cpu", seed=s) for s in (2, 5)]
    layer = moe.MoELayer(moe.config_from_workload(wl), host_io=True)
    pin = lambda t: None if t is None else t.pin_memory()
    dinp = to_device(inps[0])
    outs = []
    for inp in inps:
        out_h = torch.full((wl.T, wl.H), float("nan"), dtype=wl.torch_dtype).pin_memory()
        layer.forward_host(pin(inp.logits), pin(inp.bias), pin(inp.x), dinp.w13, dinp.w2, out_h,
                           w13_shared=dinp.w13s, w2_shared=dinp.w2s)
        outs.append(out_h)
    torch.cuda.synchronize()
    assert moe.moe_device_status(layer.ws) == 0
    for i, (inp, out_h) in enumerate(zip(inps, outs)):
        # the second input set keeps the first one's weights, as the calls did
        ref_inp = to_device(MoEInputs(logits=inp.logits, bias=inp.bias, x=inp.x, w13=inps[0].w13,
                                      w2=inps[0].w2, w13s=inps[0].w13s, w2s=inps[0].w2s))
        ref, ref_layer = _forward(wl, ref_inp, wl.n_chunks)
        if wl.reduce_dense:
            # the decode form's fp32 atomic additions come in a different order each run
            assert_float_close(storage_np(out_h), storage_np(ref), wl.dtype, f"call {i}")
        else:
            np.testing.assert_array_equal(storage_np(out_h), storage_np(ref), err_msg=f"call {i}")
    # the saved routing state is the second call's
    np.testing.assert_array_equal(layer.topk_idx.cpu().numpy(), ref_layer.topk_idx.cpu().numpy())
    np.testing.assert_array_equal(layer.keep.cpu().numpy(), ref_layer.keep.cpu().numpy())


def test_forward_host_rejects_device_activations():
    from combine_moe_route_12_b200 import moe
    wl = CASES["bf16_chunked"]
    dinp = to_device(make_inputs(wl, "cpu", seed=2))
    layer = moe.MoELayer(moe.config_from_workload(wl), host_io=True)
    out = torch.empty(wl.T, wl.H, dtype=wl.torch_dtype, device="cuda")
    with pytest.raises(ValueError):
        layer.forward_host(dinp.logits, dinp.bias, dinp.x, dinp.w13, dinp.w2, out)
    with pytest.raises(ValueError):
        moe.MoELayer(moe.config_from_workload(wl)).forward_host(None, None, None, None, None, None)


def test_nonfinite_logit_sets_status_bit():
    from combine_moe_route_12_b200 import moe
    wl = CASES["bf16_ragged_m"]
    cfg = moe.config_from_workload(wl)
    logits = torch.randn(wl.T, wl.E, device="cuda")
    logits[5, 3] = float("nan")
    ws = moe.alloc_workspace(moe.workspace_bytes(cfg))
    idx = torch.empty(wl.T, wl.k, dtype=torch.int32, device="cuda")
    w = torch.empty(wl.T, wl.k, device="cuda")
    counts = torch.empty(wl.E, dtype=torch.int32, device="cuda")
    moe.moe_route_topk(cfg, logits, None, idx, w, counts, ws)
    assert moe.moe_device_status(ws) & moe.MOE_DEV_NONFINITE_LOGIT
    assert moe.moe_device_status(ws) == 0          # read clears
    logits[5, 3] = 0.0
    moe.moe_route_topk(cfg, logits, None, idx, w, counts, ws)
    assert moe.moe_device_status(ws) == 0
    # the other tokens are still routed exactly
    oi, ow, _, _ = oracle.route_topk(logits.cpu().numpy(), None, wl.k)
    np.testing.assert_array_equal(idx.cpu().numpy(), oi)


def test_out_of_range_expert_id_is_flagged_not_written():
    from combine_moe_route_12_b200 import moe
    wl = CASES["bf16_ragged_m"]
    cfg = moe.config_from_workload(wl)
    ws = moe.alloc_workspace(moe.workspace_bytes(cfg))
    idx = torch.randint(0, wl.E, (wl.T, wl.k), dtype=torch.int32, device="cuda")
    idx[:, 1] = (idx[:, 0] + 1) % wl.E
    idx[7, 0] = wl.E + 3                           # corrupt saved state
    keep = torch.ones(wl.T, wl.k, dtype=torch.uint8, device="cuda")
    nmax = moe.max_recv_rows(cfg, wl.T)
    eoff = torch.empty(wl.E + 1, dtype=torch.int32, device="cuda")
    roff = torch.empty(wl.ep + 1, dtype=torch.int32, device="cuda")
    rt = torch.full((nmax,), -5, dtype=torch.int32, device="cuda")
    rs = torch.full((nmax,), -5, dtype=torch.int32, device="cuda")
    pos = torch.empty(wl.T, wl.k, dtype=torch.int32, device="cuda")
    spl = torch.empty(wl.ep, wl.ep, dtype=torch.int32, device="cuda")
    moe.moe_dispatch_layout(cfg, 0, wl.T, idx, keep, eoff, roff, rt, rs, pos, spl, None, ws)
    assert moe.moe_device_status(ws) & moe.MOE_DEV_BAD_INDEX
    assert pos[7, 0].item() == -1
    assert int(eoff[wl.E].item()) == wl.T * wl.k - 1
