"""GPU parity of the FP8 expert FFN (E4M3 codes with one UE8M0 scale per row)
against the oracle.

Bar: the row quantisation (codes and scales) bit-exact, for any input; the
permuted codes bit-exact; h and y, and the layer output, within the bf16 bar
(max|a-b| / max|ref| <= 2e-2; fp32 accumulation on both sides of exact E4M3
products).  h's codes come from h rounded to bf16 on both sides, from fp32
(CUDA) and fp64 (oracle) sums: a value on a rounding boundary can land one
bf16 step apart and then one code apart, so almost all (>= 99%) must be equal
and the rest within the value tolerance.  The weights' codes are the oracle's
(its quantisation of the bf16 weights), uploaded as inputs.
"""
import numpy as np
import pytest
import torch

import oracle
from combine_moe_route_12_b200 import moe
from combine_moe_route_12_b200.workload import MoEInputs, MoEWorkload, make_inputs

from moe_testlib import (assert_codes_close, assert_float_close, assert_routing_equal,
                         fp8_weights_to_device, oracle_fp8_ffn_and_out, oracle_fp8_weights,
                         oracle_routing, run_gpu_steps, storage_np, to_device)

pytestmark = pytest.mark.gpu

W = MoEWorkload
CASES = {
    # ~128 rows per expert: ragged token tiles; K = 256 (one stage) and 128
    "fp8_basic": W("fp8_basic", T=512, H=256, E=8, k=2, I=128, dtype="bf16", ep=2, ffn_fp8=True),
    # H = 384 (a stage and a half), I = 256 (two feature blocks), 16 experts
    "fp8_ragged": W("fp8_ragged", T=384, H=384, E=16, k=4, I=256, dtype="bf16", ep=4, ffn_fp8=True),
    # skewed router with a binding capacity
    "fp8_capacity": W("fp8_capacity", T=512, H=128, E=16, k=4, I=128, dtype="bf16", ep=4,
                      capacity=64, skew_bias=True, ffn_fp8=True),
    # 256 experts with ~8 rows each: the short token box
    "fp8_many_experts": W("fp8_many_experts", T=256, H=128, E=256, k=8, I=128, dtype="bf16",
                          ep=64, ffn_fp8=True),
    # four dispatch chunks
    "fp8_chunked": W("fp8_chunked", T=512, H=256, E=8, k=2, I=128, dtype="bf16", ep=2, n_chunks=4,
                     ffn_fp8=True),
    # decode: reduce straight into a dense output
    "fp8_decode": W("fp8_decode", T=64, H=256, E=32, k=8, I=128, dtype="bf16", ep=8, capacity=32,
                    reduce_dense=True, ffn_fp8=True),
}


def _special_rows(cols, rng, f32):
    rows = [np.zeros(cols), np.full(cols, -0.0)]
    r = np.zeros(cols); r[cols // 2] = -3.0; rows.append(r)                   # one nonzero
    for e in (-100, -7, 0, 9, 100):
        r = rng.normal(0, 1, cols); r[0] = 448.0 * 2.0 ** e; rows.append(r)   # scale boundary, exact
        r = rng.normal(0, 1, cols) * 2.0 ** (e - 12); r[1] = 224.0 * 2.0 ** e; rows.append(r)
    mids = oracle.e4m3_decode(np.arange(0, 0x7E, dtype=np.uint8))
    r = np.resize((mids[1:] + mids[:-1]) / 2, cols) * np.where(np.arange(cols) % 2, 1, -1)
    r[2] = 448.0; rows.append(r)                                               # every tie, scale 1
    if f32:
        r = rng.normal(0, 1, cols) * 1e-41; rows.append(r)                    # fp32 subnormals
    return np.stack(rows)


@pytest.mark.parametrize("cols,dtype", [(2048, "bf16"), (768, "bf16"), (7168, "bf16"),
                                        (136, "bf16"), (8, "bf16"), (128, "f32"), (4, "f32")])
def test_quantize_rows_bit_exact(cols, dtype):
    rng = np.random.default_rng(cols)
    f32 = dtype == "f32"
    a = rng.normal(0, 1, (97, cols)) * np.ldexp(1.0, rng.integers(-60, 60, 97))[:, None]
    a = np.concatenate([a, _special_rows(cols, rng, f32)]).astype(np.float32)
    t = torch.from_numpy(a)
    if not f32:
        t = t.to(torch.bfloat16)
    codes, scales = moe.quantize_fp8(t.cuda())
    ref_c, ref_s = oracle.quantize_rows(storage_np(t))
    np.testing.assert_array_equal(scales.cpu().numpy(), ref_s)
    np.testing.assert_array_equal(codes.cpu().numpy(), ref_c)


def test_quantize_rows_rejects_bad_arguments():
    x = torch.zeros(4, 12, dtype=torch.bfloat16, device="cuda")
    c = torch.empty(4, 12, dtype=torch.uint8, device="cuda")
    s = torch.empty(4, dtype=torch.uint8, device="cuda")
    with pytest.raises(moe.MoEError):
        moe.moe_quantize_fp8_rows(x, c, s)           # 12 bf16 columns: not a multiple of 8


def _prepare(name, seed=1):
    wl = CASES[name]
    inp = make_inputs(wl, "cpu", seed=seed)
    wq = oracle_fp8_weights(inp)
    return wl, inp, wq


@pytest.mark.parametrize("name", sorted(CASES))
def test_fp8_layer_steps_match_oracle(name):
    wl, inp, wq = _prepare(name)
    dinp = to_device(inp)
    g = run_gpu_steps(wl, dinp, fp8=fp8_weights_to_device(wq))
    assert g["status"] == 0
    orc = oracle_routing(wl, inp)
    assert_routing_equal(g, orc, wl)
    ref = oracle_fp8_ffn_and_out(wl, inp, orc, wq)
    np.testing.assert_array_equal(g["xq"], ref["xq"])
    np.testing.assert_array_equal(g["xs"], ref["xs"])
    for c, (gc, oc) in enumerate(zip(g["chunks"], ref["chunks"])):
        np.testing.assert_array_equal(gc["xr"], oc["xrq"])          # permuted codes, bitwise
        assert_float_close(gc["h"], oc["h"], "bf16", f"h chunk {c}")
        assert_codes_close(gc["hq"], gc["hs"], oc["hq"], oc["hs"], f"h codes chunk {c}")
        if not wl.reduce_dense:
            assert_float_close(gc["y"], oc["y"], "bf16", f"y chunk {c}")
    assert_float_close(storage_np(g["out"]), ref["out"], "bf16", "out")


@pytest.mark.parametrize("name", ["fp8_basic", "fp8_chunked", "fp8_decode"])
def test_fp8_forward_matches_steps(name):
    """The chunked two-stream forward in FP8 (x quantised per chunk inside it)
    gives the step path's bits; the host-buffer entry point the same."""
    wl, inp, wq = _prepare(name, seed=2)
    dinp = to_device(inp)
    w13q, w13s, w2q, w2s = fp8_weights_to_device(wq)
    layer = moe.MoELayer(moe.config_from_workload(wl), host_io=True)
    out = torch.full((wl.T, wl.H), float("nan"), dtype=torch.bfloat16, device="cuda")
    layer.forward(dinp.logits, dinp.bias, dinp.x, w13q, w2q, out, w13_scale=w13s, w2_scale=w2s)
    out_h = torch.full((wl.T, wl.H), float("nan"), dtype=torch.bfloat16).pin_memory()
    pin = lambda t: None if t is None else t.pin_memory()
    layer.forward_host(pin(inp.logits), pin(inp.bias), pin(inp.x), w13q, w2q, out_h,
                       w13_scale=w13s, w2_scale=w2s)
    torch.cuda.synchronize()
    assert moe.moe_device_status(layer.ws) == 0
    g = run_gpu_steps(wl, dinp, fp8=(w13q, w13s, w2q, w2s))
    if wl.reduce_dense:
        assert_float_close(storage_np(out), storage_np(g["out"]), "bf16", "forward")
        assert_float_close(storage_np(out_h), storage_np(g["out"]), "bf16", "forward_host")
    else:
        np.testing.assert_array_equal(storage_np(out), storage_np(g["out"]))
        np.testing.assert_array_equal(storage_np(out_h), storage_np(g["out"]))
    orc = oracle_routing(wl, inp)
    ref = oracle_fp8_ffn_and_out(wl, inp, orc, wq)
    assert_float_close(storage_np(out), ref["out"], "bf16", "out vs oracle")


def test_fp8_forward_needs_scales_and_rejects_shared_expert():
    wl = CASES["fp8_basic"]
    cfg = moe.config_from_workload(wl)
    layer = moe.MoELayer(cfg)
    z = torch.zeros(1, device="cuda")
    with pytest.raises(moe.MoEError):
        layer.forward(z, None, z, z, z, z)
    with pytest.raises(moe.MoEError):
        moe.config_check(moe.config_from_workload(wl.with_(shared_I=128)))
    with pytest.raises(moe.MoEError):
        moe.config_check(moe.config_from_workload(wl.with_(H=192)))


@pytest.mark.parametrize("name", ["fp8_basic", "fp8_capacity", "fp8_many_experts", "fp8_chunked"])
def test_permute_quantize_equals_quantize_then_permute(name):
    """The fused form writes the oracle's codes (its row quantisation followed by
    its permute) to the receive rows, and the oracle's scales for every token
    that keeps a slot; rows and scales of other tokens stay untouched."""
    wl, inp, wq = _prepare(name, seed=4)
    dinp = to_device(inp)
    g = run_gpu_steps(wl, dinp, fp8=fp8_weights_to_device(wq))
    orc = oracle_routing(wl, inp)
    assert_routing_equal(g, orc, wl)
    xq_ref, xs_ref = oracle.quantize_rows(storage_np(inp.x))
    cfg = moe.config_from_workload(wl)
    tc = wl.T // wl.n_chunks
    nmax = moe.max_recv_rows(cfg, tc)
    xs = torch.full((wl.T,), 0xEE, dtype=torch.uint8, device="cuda")
    for c, gc in enumerate(g["chunks"]):
        pos = torch.from_numpy(gc["pos"]).cuda()
        xr = torch.full((max(nmax, 1), wl.H), 0xEE, dtype=torch.uint8, device="cuda")
        moe.moe_permute_quantize_fp8(cfg, dinp.x, pos, c * tc, tc, xr, xs)
        torch.cuda.synchronize()
        lay = orc["layouts"][c]
        n = lay["N"]
        np.testing.assert_array_equal(xr[:n].cpu().numpy(), oracle.permute(xq_ref, lay["recv_token"]))
        assert (xr[n:].cpu().numpy() == 0xEE).all()
    kept_tok = orc["keep"].any(axis=1)
    np.testing.assert_array_equal(xs.cpu().numpy()[kept_tok], xs_ref[kept_tok])
    assert (xs.cpu().numpy()[~kept_tok] == 0xEE).all()


def test_permute_quantize_rejects_long_rows():
    cfg = moe.config_from_workload(CASES["fp8_basic"].with_(H=8320))
    z = torch.zeros(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(moe.MoEError):
        moe.moe_permute_quantize_fp8(cfg, z, z, 0, 0, z, z)
