"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times.

Routing, drop sets, layouts and split counts are compared whole against the
oracle (bit-exact).  Permuted rows are checked whole by the defining property
xr[p] = x[recv_token[p]] (bitwise).  The FFN and the combined output are
compared on sampled rows and tokens that the oracle computes one by one:
experts at both ends of the expert range, the most loaded expert and a random
one, each with its first, last and random rows; and tokens spread over the
batch.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_moe_route_12_b200 import moe
from combine_moe_route_12_b200.workload import WORKLOADS, MoEInputs, make_inputs

from moe_testlib import (assert_codes_close, assert_float_close, assert_routing_equal,
                         oracle_fp8_weights, oracle_routing, run_gpu_steps, storage_np)

pytestmark = pytest.mark.gpu

FULL = ["qwen3_30b_a3b", "skew_capacity", "dsv3_prefill", "dsv3_decode", "dsv3_grouped"]


def _host_expert(inp, e, cache):
    if e not in cache:
        cache[e] = (storage_np(inp.w13[e]), storage_np(inp.w2[e]))
    return cache[e]


@pytest.mark.parametrize("name", FULL)
def test_fullsize_against_oracle(name):
    wl = WORKLOADS[name]
    torch.cuda.empty_cache()
    inp = make_inputs(wl, "cuda")
    g = run_gpu_steps(wl, inp, keep_rows=False)
    assert g["status"] == 0
    cpu_inp = MoEInputs(logits=inp.logits.cpu(), bias=None if inp.bias is None else inp.bias.cpu(),
                        x=inp.x.cpu(), w13=inp.w13, w2=inp.w2)
    orc = oracle_routing(wl, cpu_inp)
    assert_routing_equal(g, orc, wl)
    if wl.capacity >= 0:
        assert (orc["kept_counts"] <= wl.capacity).all()

    x_np = storage_np(inp.x)
    rng = np.random.default_rng(0)
    cache = {}
    for c, (gc, lay) in enumerate(zip(g["chunks"], orc["layouts"])):
        n = lay["N"]
        rt = torch.from_numpy(lay["recv_token"]).long().cuda()
        assert torch.equal(gc["xr_dev"][:n], inp.x[rt]), "permute must copy rows bitwise"
        eoff = lay["expert_offsets"]
        sizes = np.diff(eoff)
        nonempty = np.nonzero(sizes)[0]
        experts = {int(nonempty[0]), int(nonempty[-1]), int(np.argmax(sizes)),
                   int(rng.choice(nonempty))}
        for e in sorted(experts):
            lo, hi = int(eoff[e]), int(eoff[e + 1])
            rows = sorted({lo, hi - 1, *rng.integers(lo, hi, 2).tolist()})
            w13e, w2e = _host_expert(inp, e, cache)
            for p in rows:
                h_ref, y_ref, ye_ref = oracle.ffn_row(x_np[lay["recv_token"][p]], w13e, w2e)
                assert_float_close(storage_np(gc["h_dev"][p]), h_ref, wl.dtype, f"h[{p}] expert {e}")
                if gc["y_dev"] is not None:
                    assert_float_close(storage_np(gc["y_dev"][p]), y_ref, wl.dtype, f"y[{p}] expert {e}")

    out = storage_np(g["out"])
    tokens = sorted({0, wl.T - 1, *rng.integers(0, wl.T, 2).tolist()})
    shared = None
    if wl.shared_I > 0:
        shared = (storage_np(inp.w13s), storage_np(inp.w2s))
    tc = wl.T // wl.n_chunks
    for t in tokens:
        ysh = None
        if shared is not None:
            # the shared expert's row of token t, checked against the GPU's and used below
            _, ysh, _ = oracle.shared_expert(x_np[t:t + 1], *shared)
            gys = storage_np(g["chunks"][t // tc]["ys_dev"][t % tc:t % tc + 1])
            assert_float_close(gys, ysh, wl.dtype, f"y_shared[{t}]")
        ys, yes, pos = [], [], []
        for j in range(wl.k):
            if not orc["keep"][t, j]:
                pos.append(-1)
                continue
            w13e, w2e = _host_expert(inp, int(orc["topk_idx"][t, j]), cache)
            _, y_ref, ye_ref = oracle.ffn_row(x_np[t], w13e, w2e)
            pos.append(len(ys))
            ys.append(y_ref)
            yes.append(ye_ref)
        posa = np.array([pos], np.int32)
        w_t = orc["topk_w"][t:t + 1]
        if not ys:
            ref = np.zeros((1, wl.H), x_np.dtype) if ysh is None else ysh
        elif wl.reduce_dense:
            ref = oracle.combine_exact(np.stack(yes), posa, w_t, 1, x_np.dtype, y_shared=ysh)
        else:
            ref = oracle.combine(np.stack(ys), posa, w_t, 1, y_shared=ysh)
        assert_float_close(out[t:t + 1], ref, wl.dtype, f"out[{t}]")
    del g, inp
    torch.cuda.empty_cache()


def test_dsv3_prefill_chunked_forward_equals_steps():
    """Two-stream chunked forward at the full DeepSeek-V3 prefill shape gives
    the same bits as the step-by-step path, and as the unchunked forward."""
    wl = WORKLOADS["dsv3_prefill"]
    torch.cuda.empty_cache()
    inp = make_inputs(wl, "cuda", seed=3)
    g = run_gpu_steps(wl, inp, keep_rows=False)
    ref = g["out"]
    del g
    outs = []
    for n_chunks in (2, 1):
        w = wl.with_(n_chunks=n_chunks)
        layer = moe.MoELayer(moe.config_from_workload(w))
        out = torch.empty(wl.T, wl.H, dtype=wl.torch_dtype, device="cuda")
        layer.forward(inp.logits, inp.bias, inp.x, inp.w13, inp.w2, out)
        torch.cuda.synchronize()
        assert moe.moe_device_status(layer.ws) == 0
        outs.append(out)
        del layer
    assert torch.equal(outs[0], ref)
    assert torch.equal(outs[1], ref)


@pytest.mark.parametrize("name", ["qwen3_30b_a3b_fp8", "dsv3_prefill_fp8"])
def test_fp8_fullsize_against_oracle(name):
    """The FP8 layer at full size: x's codes and scales whole and bit-exact,
    the weight codes of the sampled experts bit-exact, permuted codes by the
    defining property, sampled FFN rows and tokens against the oracle's FP8
    rows (its own quantisation of the bf16 weights)."""
    wl = WORKLOADS[name]
    torch.cuda.empty_cache()
    inp = make_inputs(wl, "cuda")
    w13q, w13s = moe.quantize_fp8(inp.w13)
    w2q, w2s = moe.quantize_fp8(inp.w2)
    g = run_gpu_steps(wl, inp, keep_rows=False, fp8=(w13q, w13s, w2q, w2s))
    assert g["status"] == 0
    cpu_inp = MoEInputs(logits=inp.logits.cpu(), bias=None if inp.bias is None else inp.bias.cpu(),
                        x=inp.x.cpu(), w13=inp.w13, w2=inp.w2)
    orc = oracle_routing(wl, cpu_inp)
    assert_routing_equal(g, orc, wl)
    xq, xs = oracle.quantize_rows(storage_np(inp.x))
    np.testing.assert_array_equal(g["xq"], xq)
    np.testing.assert_array_equal(g["xs"], xs)
    xq_dev = torch.from_numpy(xq).cuda()
    rng = np.random.default_rng(0)
    cache = {}

    def expert(e):
        if e not in cache:
            cache[e] = oracle_fp8_weights(inp, [e])[e]
            ref = cache[e]
            np.testing.assert_array_equal(w13q[e].cpu().numpy(), ref["w13q"])
            np.testing.assert_array_equal(w13s[e].cpu().numpy(), ref["w13s"])
            np.testing.assert_array_equal(w2q[e].cpu().numpy(), ref["w2q"])
            np.testing.assert_array_equal(w2s[e].cpu().numpy(), ref["w2s"])
        return cache[e]

    def row(p_token, e):
        w = expert(e)
        return oracle.ffn_row_fp8(xq[p_token], xs[p_token], w["w13q"], w["w13s"], w["w2q"], w["w2s"])

    for c, (gc, lay) in enumerate(zip(g["chunks"], orc["layouts"])):
        n = lay["N"]
        rt = torch.from_numpy(lay["recv_token"]).long().cuda()
        assert torch.equal(gc["xr_dev"][:n], xq_dev[rt]), "permute must copy the code rows bitwise"
        eoff = lay["expert_offsets"]
        sizes = np.diff(eoff)
        nonempty = np.nonzero(sizes)[0]
        experts = {int(nonempty[0]), int(nonempty[-1]), int(np.argmax(sizes)), int(rng.choice(nonempty))}
        for e in sorted(experts):
            lo, hi = int(eoff[e]), int(eoff[e + 1])
            for p in sorted({lo, hi - 1, *rng.integers(lo, hi, 2).tolist()}):
                h, hq, hs, y, ye = row(int(lay["recv_token"][p]), e)
                assert_float_close(storage_np(gc["h_dev"][p]), h, "bf16", f"h[{p}] expert {e}")
                assert_codes_close(gc["hq_dev"][p:p + 1].cpu().numpy(), gc["hs_dev"][p:p + 1].cpu().numpy(),
                                   hq[None], np.array([hs], np.uint8), f"h codes[{p}]", min_equal=0.98)
                assert_float_close(storage_np(gc["y_dev"][p]), y, "bf16", f"y[{p}] expert {e}")

    out = storage_np(g["out"])
    for t in sorted({0, wl.T - 1, *rng.integers(0, wl.T, 2).tolist()}):
        ys, pos = [], []
        for j in range(wl.k):
            if not orc["keep"][t, j]:
                pos.append(-1)
                continue
            pos.append(len(ys))
            ys.append(row(t, int(orc["topk_idx"][t, j]))[3])
        ref = oracle.combine(np.stack(ys), np.array([pos], np.int32), orc["topk_w"][t:t + 1], 1)
        assert_float_close(out[t:t + 1], ref, "bf16", f"out[{t}]")
    del g, inp
    torch.cuda.empty_cache()
