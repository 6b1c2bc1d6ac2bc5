"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times.

Routing, drop sets, layouts and split counts are compared whole against the
oracle (bit-exact).  Permuted rows are checked whole by the defining property
xr[p] = x[recv_token[p]] (bitwise).  The FFN is compared on every tile the
grouped GEMM deals, at both sides of every boundary inside it: an expert's rows
in 256-token tiles, the last one of up to 288 (its main MMA of N <= 256 split
between the two CTAs of the pair, the rows past 256 in a second MMA split the
same way), so per tile its first and last row and the rows on either side of
each CTA half; two more rows of each short tile (the 32-row token box of tiles
with at most 64 rows).  The combined output is
compared on 128 sampled tokens, whose expert rows the oracle also computes.
The oracle's rows run in threads (its C calls release the interpreter lock),
expert by expert, each with its own host copy of that expert's weights.
"""
import concurrent.futures as cf
import os

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


TILE = 256          # token rows per FFN tile (an expert's last takes up to TILE_MAX)
TILE_MAX = 288
MX_TILE = 224       # token rows per tile of the block-scaled FP8 FFN
SHORT = 64          # tiles of at most this many rows take the short token box
N_TOKENS = 128      # sampled tokens of the combined output


def ffn_tiles(m):
    """(first row, rows, main MMA N, extra MMA N) of the FFN's tiles over an expert
    of m rows: 256-row tiles, the last one of up to 288."""
    if m <= 0:
        return []
    n = 1 if m <= TILE_MAX else (m - (TILE_MAX - TILE) + TILE - 1) // TILE
    out = []
    for t in range(n):
        nv = m - t * TILE if t == n - 1 else TILE
        n_main = TILE if nv > 224 else (nv + 15) // 16 * 16
        out.append((t * TILE, nv, n_main, 32 if nv > TILE else 0))
    return out


def mx_tiles(m):
    """The block-scaled FFN's tiles over an expert of m rows: 224 rows each (its MMA
    N rounded to 16, split between the two CTAs)."""
    return [(r0, min(MX_TILE, m - r0), (min(MX_TILE, m - r0) + 15) // 16 * 16, 0)
            for r0 in range(0, m, MX_TILE)]


def select_rows(lay, rng, tiles=None, short=SHORT):
    """Receive rows that cover every FFN tile of a chunk, following the kernel's
    tiling (tiles: rows -> [(first row, rows, main N, extra N)], the bf16 / FP8
    kernel's by default): per tile its first and last row and the rows on either
    side of each CTA half of its main and extra MMA; a short tile (<= short rows)
    two more."""
    tiles = tiles or ffn_tiles
    eoff = lay["expert_offsets"]
    rows = set()
    for e in range(len(eoff) - 1):
        lo, hi = int(eoff[e]), int(eoff[e + 1])
        for r0, nv, n_main, n_x in tiles(hi - lo):
            a, b = n_main // 2, n_x // 2
            edges = {0, a - 1, a, a + b - 1, a + b, 2 * a + b - 1, 2 * a + b, nv - 1}
            rows.update(lo + r0 + r for r in edges if 0 <= r < nv)
            if nv <= short:
                rows.update(int(v) for v in rng.integers(lo + r0, lo + r0 + nv, 2))
    return rows


def expert_of(eoff, p):
    return int(np.searchsorted(eoff, p, side="right") - 1)


def oracle_rows(row_fn, fetch, wanted):
    """wanted: {expert: [(key, x_row), ...]} -> {key: row_fn(x_row, weights)}, run
    expert by expert in threads."""
    def work(e, items):
        w = fetch(e)
        return [(key, row_fn(xv, w)) for key, xv in items]
    out = {}
    n = max(1, min(32, os.cpu_count() or 1))
    with cf.ThreadPoolExecutor(n) as ex:
        for res in ex.map(lambda kv: work(*kv), wanted.items()):
            out.update(res)
    return out


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
    tc = wl.T // wl.n_chunks
    tokens = sorted({0, wl.T - 1, *rng.choice(wl.T, N_TOKENS - 2, replace=False).tolist()})
    # every tile's rows, and the rows of the sampled tokens' kept slots
    wanted = {}
    for c, lay in enumerate(orc["layouts"]):
        n = lay["N"]
        rt = torch.from_numpy(lay["recv_token"]).long().cuda()
        assert torch.equal(g["chunks"][c]["xr_dev"][:n], inp.x[rt]), "permute must copy rows bitwise"
        rows = select_rows(lay, rng)
        for t in tokens:
            if c * tc <= t < (c + 1) * tc:
                rows.update(int(p) for p in lay["pos"][t - c * tc] if p >= 0)
        for p in rows:
            e = expert_of(lay["expert_offsets"], p)
            wanted.setdefault(e, []).append(((c, p), x_np[lay["recv_token"][p]]))
    fetch = lambda e: (storage_np(inp.w13[e]), storage_np(inp.w2[e]))
    ref = oracle_rows(lambda xv, w: oracle.ffn_row(xv, w[0], w[1]), fetch, wanted)

    assert len(ref) == sum(len(v) for v in wanted.values())
    for (c, p), (h_ref, y_ref, _) in sorted(ref.items()):
        gc = g["chunks"][c]
        assert_float_close(storage_np(gc["h_dev"][p]), h_ref, wl.dtype, f"h[{p}] chunk {c}")
        if gc["y_dev"] is not None:
            assert_float_close(storage_np(gc["y_dev"][p]), y_ref, wl.dtype, f"y[{p}] chunk {c}")

    out = storage_np(g["out"])
    shared = None
    if wl.shared_I > 0:
        shared = (storage_np(inp.w13s), storage_np(inp.w2s))
    for t in tokens:
        c = t // tc
        lay = orc["layouts"][c]
        ysh = None
        if shared is not None:
            # the shared expert's row of token t, checked against the GPU's and used below
            _, ysh, _ = oracle.shared_expert(x_np[t:t + 1], *shared)
            gys = storage_np(g["chunks"][c]["ys_dev"][t % tc:t % tc + 1])
            assert_float_close(gys, ysh, wl.dtype, f"y_shared[{t}]")
        ys, yes, pos = [], [], []
        for j in range(wl.k):
            p = int(lay["pos"][t - c * tc, j])
            if p < 0:
                pos.append(-1)
                continue
            _, y_ref, ye_ref = ref[(c, p)]
            pos.append(len(ys))
            ys.append(y_ref)
            yes.append(ye_ref)
        posa = np.array([pos], np.int32)
        w_t = orc["topk_w"][t:t + 1]
        if not ys:
            want = np.zeros((1, wl.H), x_np.dtype) if ysh is None else ysh
        elif wl.reduce_dense:
            want = oracle.combine_exact(np.stack(yes), posa, w_t, 1, x_np.dtype, y_shared=ysh)
        else:
            want = oracle.combine(np.stack(ys), posa, w_t, 1, y_shared=ysh)
        assert_float_close(out[t:t + 1], want, wl.dtype, f"out[{t}]")
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
    the weight codes of every checked expert bit-exact, permuted codes by the
    defining property, the rows of every FFN tile and 128 sampled tokens
    against the oracle's FP8 rows (its own quantisation of the bf16 weights)."""
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

    def fetch(e):
        # the oracle's codes of expert e's weights, checked against the GPU's
        ref = oracle_fp8_weights(inp, [e])[e]
        np.testing.assert_array_equal(w13q[e].cpu().numpy(), ref["w13q"])
        np.testing.assert_array_equal(w13s[e].cpu().numpy(), ref["w13s"])
        np.testing.assert_array_equal(w2q[e].cpu().numpy(), ref["w2q"])
        np.testing.assert_array_equal(w2s[e].cpu().numpy(), ref["w2s"])
        return ref

    tc = wl.T // wl.n_chunks
    tokens = sorted({0, wl.T - 1, *rng.choice(wl.T, N_TOKENS - 2, replace=False).tolist()})
    wanted = {}
    for c, (gc, lay) in enumerate(zip(g["chunks"], orc["layouts"])):
        n = lay["N"]
        rt = torch.from_numpy(lay["recv_token"]).long().cuda()
        assert torch.equal(gc["xr_dev"][:n], xq_dev[rt]), "permute must copy the code rows bitwise"
        rows = select_rows(lay, rng)
        for t in tokens:
            if c * tc <= t < (c + 1) * tc:
                rows.update(int(p) for p in lay["pos"][t - c * tc] if p >= 0)
        for p in rows:
            e = expert_of(lay["expert_offsets"], p)
            wanted.setdefault(e, []).append(((c, p), int(lay["recv_token"][p])))
    ref = oracle_rows(lambda tok, w: oracle.ffn_row_fp8(xq[tok], xs[tok], w["w13q"], w["w13s"], w["w2q"],
                                                        w["w2s"]), fetch, wanted)
    assert len(ref) == sum(len(v) for v in wanted.values())
    for (c, p), (h, hq, hs, y, ye) in sorted(ref.items()):
        gc = g["chunks"][c]
        assert_float_close(storage_np(gc["h_dev"][p]), h, "bf16", f"h[{p}] chunk {c}")
        assert_codes_close(gc["hq_dev"][p:p + 1].cpu().numpy(), gc["hs_dev"][p:p + 1].cpu().numpy(),
                           hq[None], np.array([hs], np.uint8), f"h codes[{p}]", min_equal=0.98)
        assert_float_close(storage_np(gc["y_dev"][p]), y, "bf16", f"y[{p}] chunk {c}", per_element=False)

    out = storage_np(g["out"])
    for t in tokens:
        c = t // tc
        lay = orc["layouts"][c]
        ys, pos = [], []
        for j in range(wl.k):
            p = int(lay["pos"][t - c * tc, j])
            if p < 0:
                pos.append(-1)
                continue
            pos.append(len(ys))
            ys.append(ref[(c, p)][3])
        want = oracle.combine(np.stack(ys), np.array([pos], np.int32), orc["topk_w"][t:t + 1], 1)
        assert_float_close(out[t:t + 1], want, "bf16", f"out[{t}]", per_element=False)
    del g, inp
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["qwen3_30b_a3b_mxfp8", "dsv3_prefill_mxfp8"])
def test_mxfp8_fullsize_against_oracle(name):
    """The FP8 layer with K-blocked scales at full size: x's block quantisation
    whole and bit-exact (the standalone kernel), the fused permute's codes and
    scales whole by the defining property (xr[p] = q(x)[recv_token[p]]), every
    checked expert's weight codes and scales bit-exact, the rows at every boundary
    of every 224-row FFN tile and of 128 sampled tokens against the oracle's blocked FP8
    rows (h's codes by the adjacency bar, y by the bf16 bar), and the combined
    output of those tokens."""
    wl = WORKLOADS[name]
    torch.cuda.empty_cache()
    inp = make_inputs(wl, "cuda")
    w13q, w13s = moe.quantize_fp8_blocks(inp.w13)
    w2q, w2s = moe.quantize_fp8_blocks(inp.w2)
    g = run_gpu_steps(wl, inp, keep_rows=False, fp8=(w13q, w13s, w2q, w2s))
    assert g["status"] == 0
    cpu_inp = MoEInputs(logits=inp.logits.cpu(), bias=None if inp.bias is None else inp.bias.cpu(),
                        x=inp.x.cpu(), w13=inp.w13, w2=inp.w2)
    orc = oracle_routing(wl, cpu_inp)
    assert_routing_equal(g, orc, wl)
    xq, xs = oracle.quantize_blocks(storage_np(inp.x), 32)
    gxq, gxs = moe.quantize_fp8_blocks(inp.x)
    np.testing.assert_array_equal(gxq.cpu().numpy(), xq)
    np.testing.assert_array_equal(gxs.cpu().numpy(), xs)
    xq_dev, xs_dev = torch.from_numpy(xq).cuda(), torch.from_numpy(xs).cuda()
    del gxq, gxs
    rng = np.random.default_rng(0)
    H, I = wl.H, wl.I

    def fetch(e):
        # the oracle's block codes of expert e's weights, checked against the GPU's
        a13, s13 = oracle.quantize_blocks(storage_np(inp.w13[e]), 32)
        a2, s2 = oracle.quantize_blocks(storage_np(inp.w2[e]), 32)
        np.testing.assert_array_equal(w13q[e].cpu().numpy().reshape(a13.shape), a13)
        np.testing.assert_array_equal(w13s[e].cpu().numpy().reshape(s13.shape), s13)
        np.testing.assert_array_equal(w2q[e].cpu().numpy().reshape(a2.shape), a2)
        np.testing.assert_array_equal(w2s[e].cpu().numpy().reshape(s2.shape), s2)
        return a13, s13, a2, s2

    tc = wl.T // wl.n_chunks
    tokens = sorted({0, wl.T - 1, *rng.choice(wl.T, N_TOKENS - 2, replace=False).tolist()})
    wanted = {}
    for c, (gc, lay) in enumerate(zip(g["chunks"], orc["layouts"])):
        n = lay["N"]
        rt = torch.from_numpy(lay["recv_token"]).long().cuda()
        assert torch.equal(gc["xr_dev"][:n], xq_dev[rt]), "fused permute: codes"
        assert torch.equal(gc["xsf_dev"][:n], xs_dev[rt]), "fused permute: block scales"
        rows = select_rows(lay, rng, tiles=mx_tiles, short=0)
        for t in tokens:
            if c * tc <= t < (c + 1) * tc:
                rows.update(int(p) for p in lay["pos"][t - c * tc] if p >= 0)
        for p in rows:
            e = expert_of(lay["expert_offsets"], p)
            wanted.setdefault(e, []).append(((c, p), int(lay["recv_token"][p])))
    ref = oracle_rows(lambda tok, w: oracle.ffn_row_fp8_blocked(xq[tok], xs[tok], *w, 32), fetch, wanted)
    assert len(ref) == sum(len(v) for v in wanted.values())
    keys = sorted(ref)
    for c in range(wl.n_chunks):
        ps = [p for cc, p in keys if cc == c]
        if not ps:
            continue
        gc = g["chunks"][c]
        sel = torch.tensor(ps, dtype=torch.long, device="cuda")
        ghq, ghs = gc["hq_dev"][sel].cpu().numpy(), gc["hsf_dev"][sel].cpu().numpy()
        rhq = np.stack([ref[(c, p)][1] for p in ps])
        rhs = np.stack([ref[(c, p)][2] for p in ps])
        assert_codes_close(ghq, ghs.reshape(-1), rhq, rhs.reshape(-1), f"h codes chunk {c}")
        gy = storage_np(gc["y_dev"][sel])
        for j, p in enumerate(ps):
            assert_float_close(gy[j], ref[(c, p)][3], "bf16", f"y[{p}] chunk {c}", per_element=False)

    out = storage_np(g["out"])
    for t in tokens:
        c = t // tc
        lay = orc["layouts"][c]
        ys, pos = [], []
        for j in range(wl.k):
            p = int(lay["pos"][t - c * tc, j])
            if p < 0:
                pos.append(-1)
                continue
            pos.append(len(ys))
            ys.append(ref[(c, p)][3])
        want = oracle.combine(np.stack(ys), np.array([pos], np.int32), orc["topk_w"][t:t + 1], 1)
        assert_float_close(out[t:t + 1], want, "bf16", f"out[{t}]", per_element=False)
    del g, inp
    torch.cuda.empty_cache()
