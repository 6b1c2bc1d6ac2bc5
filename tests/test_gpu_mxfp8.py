"""GPU parity of the FP8 expert FFN with K-blocked UE8M0 scales (cfg.ffn_fp8 = 2:
one scale per row and 32 K values, h quantised inside GEMM1's SwiGLU epilogue)
against the oracle's blocked FP8 row (LightLLM PR 1687: the FP8 grouped GEMM with
UE8M0 scales packed four to an int32; silu_and_mul followed by the quantisation
of h).

Bar: the block quantisation (codes and scales) of x and of the weights bit-exact;
the permuted codes and their per-receive-row scales bit-exact; h's codes and
scales come from h summed in fp32 (GPU) or fp64 (oracle) and rounded to bf16, so
>= 99 % equal and every differing code a neighbour of the oracle's; y and out
within the bf16 bar against the oracle's rows (computed from its own h codes).
"""
import numpy as np
import pytest
import torch

import oracle
from combine_moe_route_12_b200 import moe
from combine_moe_route_12_b200.workload import MoEWorkload, make_inputs

from moe_testlib import (assert_codes_close, assert_float_close, assert_routing_equal,
                         oracle_routing, run_gpu_steps, storage_np)

pytestmark = pytest.mark.gpu

W = MoEWorkload
CASES = {
    # one ring stage per GEMM (K = 256), ragged experts
    "mx_ragged": W("mx_ragged", T=512, H=256, E=8, k=2, I=256, dtype="bf16", ep=2, ffn_fp8=2),
    # K = 128: the single stage is half past K (zero codes, zero scale words)
    "mx_k128": W("mx_k128", T=256, H=128, E=4, k=2, I=128, dtype="bf16", ep=2, ffn_fp8=2),
    # three stages of H, one and a half of I, a binding capacity with skew
    "mx_long_k": W("mx_long_k", T=512, H=768, E=8, k=2, I=384, dtype="bf16", ep=2, capacity=100,
                   skew_bias=True, ffn_fp8=2),
    # many experts (short tiles), two chunks
    "mx_many_experts": W("mx_many_experts", T=2048, H=256, E=128, k=4, I=128, dtype="bf16", ep=4,
                         n_chunks=2, ffn_fp8=2),
    # experts with several 128-token blocks
    "mx_token_blocks": W("mx_token_blocks", T=1024, H=256, E=4, k=2, I=256, dtype="bf16", ep=2, ffn_fp8=2),
    # decode form: fp32 reduce of w * y
    "mx_decode": W("mx_decode", T=128, H=256, E=16, k=4, I=256, dtype="bf16", ep=4, capacity=64,
                   reduce_dense=True, ffn_fp8=2),
}


def _quantized_weights(inp):
    w13q, w13s = moe.quantize_fp8_blocks(inp.w13)
    w2q, w2s = moe.quantize_fp8_blocks(inp.w2)
    return w13q, w13s, w2q, w2s


@pytest.mark.parametrize("dtype,rows,cols", [("bf16", 37, 256), ("bf16", 5, 7168), ("f32", 9, 96)])
def test_block_quantisation_bit_exact(dtype, rows, cols):
    g = torch.Generator().manual_seed(rows)
    a = torch.randn(rows, cols, generator=g) * torch.exp2(torch.randint(-30, 30, (rows, 1), generator=g).float())
    a[:, 32:64] *= 1e-6                     # a quiet block takes its own scale
    a[0, :32] = 0                           # a zero block
    a = a.to(torch.bfloat16 if dtype == "bf16" else torch.float32)
    codes, scales = moe.quantize_fp8_blocks(a.cuda())
    ref_c, ref_s = oracle.quantize_blocks(storage_np(a), 32)
    np.testing.assert_array_equal(codes.cpu().numpy(), ref_c)
    np.testing.assert_array_equal(scales.cpu().numpy(), ref_s)


@pytest.mark.parametrize("name", sorted(CASES))
def test_mxfp8_layer_steps_match_oracle(name):
    wl = CASES[name]
    inp = make_inputs(wl, "cuda", seed=2)
    w13q, w13s, w2q, w2s = _quantized_weights(inp)
    g = run_gpu_steps(wl, inp, fp8=(w13q, w13s, w2q, w2s))
    assert g["status"] == 0
    orc = oracle_routing(wl, inp)
    assert_routing_equal(g, orc, wl)
    # the weights' block quantisation, bit-exact
    ow13q, ow13s = oracle.quantize_blocks(storage_np(inp.w13).reshape(-1, wl.H), 32)
    ow2q, ow2s = oracle.quantize_blocks(storage_np(inp.w2).reshape(-1, wl.I), 32)
    np.testing.assert_array_equal(w13q.cpu().numpy().reshape(ow13q.shape), ow13q)
    np.testing.assert_array_equal(w13s.cpu().numpy().reshape(ow13s.shape), ow13s)
    np.testing.assert_array_equal(w2q.cpu().numpy().reshape(ow2q.shape), ow2q)
    np.testing.assert_array_equal(w2s.cpu().numpy().reshape(ow2s.shape), ow2s)
    ow13q = ow13q.reshape(wl.E, 2 * wl.I, wl.H)
    ow13s = ow13s.reshape(wl.E, 2 * wl.I, wl.H // 32)
    ow2q = ow2q.reshape(wl.E, wl.H, wl.I)
    ow2s = ow2s.reshape(wl.E, wl.H, wl.I // 32)
    xq, xs = oracle.quantize_blocks(storage_np(inp.x), 32)
    out_ref = np.zeros((wl.T, wl.H), np.uint16)
    tc = wl.T // wl.n_chunks
    for c, (gc, lay) in enumerate(zip(g["chunks"], orc["layouts"])):
        n = lay["N"]
        rt = lay["recv_token"]
        np.testing.assert_array_equal(gc["xr"], xq[rt], err_msg="permuted codes")
        np.testing.assert_array_equal(gc["xsf"], xs[rt], err_msg="permuted block scales")
        eoff = lay["expert_offsets"]
        hq = np.zeros((n, wl.I), np.uint8)
        hs = np.zeros((n, wl.I // 32), np.uint8)
        y = np.zeros((n, wl.H), np.uint16)
        ye = np.zeros((n, wl.H), np.float64)
        for e in range(wl.E):
            for p in range(int(eoff[e]), int(eoff[e + 1])):
                t = int(rt[p])
                _, hq[p], hs[p], y[p], ye[p] = oracle.ffn_row_fp8_blocked(
                    xq[t], xs[t], ow13q[e], ow13s[e], ow2q[e], ow2s[e], 32)
        if n:
            assert_codes_close(gc["hq"], gc["hsf"].reshape(-1), hq, hs.reshape(-1), f"h codes chunk {c}")
        if gc["y"] is not None:
            assert_float_close(gc["y"], y, "bf16", f"y chunk {c}", per_element=False)
        if wl.reduce_dense:
            oracle.combine_exact(ye, lay["pos"], orc["topk_w"], wl.T, np.uint16, c * tc, out_ref)
        else:
            oracle.combine(y, lay["pos"], orc["topk_w"], wl.T, c * tc, out_ref)
    assert_float_close(storage_np(g["out"]), out_ref, "bf16", "out", per_element=False)


@pytest.mark.parametrize("name", ["mx_many_experts", "mx_decode"])
def test_mxfp8_forward_equals_steps(name):
    """The chunked forward (both streams) and the host-buffer forward with
    ffn_fp8 = 2 against the step path: the same bits (the decode form up to the
    order of its fp32 atomic additions)."""
    wl = CASES[name]
    inp = make_inputs(wl, "cuda", seed=4)
    w13q, w13s, w2q, w2s = _quantized_weights(inp)
    g = run_gpu_steps(wl, inp, fp8=(w13q, w13s, w2q, w2s))
    cfg = moe.config_from_workload(wl)
    layer = moe.MoELayer(cfg, host_io=True)
    out = torch.empty(wl.T, wl.H, dtype=torch.bfloat16, device="cuda")
    layer.forward(inp.logits, inp.bias, inp.x, w13q, w2q, out, w13_scale=w13s, w2_scale=w2s)
    out_h = torch.empty(wl.T, wl.H, dtype=torch.bfloat16).pin_memory()
    bias_h = None if inp.bias is None else inp.bias.cpu().pin_memory()
    layer.forward_host(inp.logits.cpu().pin_memory(), bias_h, inp.x.cpu().pin_memory(), w13q, w2q, out_h,
                       w13_scale=w13s, w2_scale=w2s)
    torch.cuda.synchronize()
    assert moe.moe_device_status(layer.ws) == 0
    if wl.reduce_dense:
        assert_float_close(storage_np(out), storage_np(g["out"]), "bf16", "forward")
        assert_float_close(storage_np(out_h), storage_np(g["out"]), "bf16", "forward_host")
    else:
        assert torch.equal(out, g["out"])
        assert torch.equal(out_h, g["out"].cpu())
