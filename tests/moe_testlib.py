"""Helpers shared by the GPU parity tests: run every ABI step of the CUDA path
on one set of inputs, run the CPU oracle on the same inputs, and compare.

Tolerances (from the layer's stated contract): indices, drop sets, layouts,
split counts, routing weights and permuted rows bit-exact; floating outputs
within max-abs 1e-4 (fp32) or max|a-b| / max|ref| <= 2e-2 (bf16, fp32
accumulate), with for bf16 also ||a-b||_2 / ||ref||_2 <= 2e-2 and at most 0.5 %
of the elements with |ref| > rms(ref) past 2e-2 of their own value.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from combine_moe_route_12_b200 import moe
from combine_moe_route_12_b200.workload import MoEInputs, MoEWorkload

F32_ABS_TOL = 1e-4
BF16_REL_TOL = 2e-2
SIGNIFICANT_FRAC = 5e-3   # bf16: share of |ref| > rms(ref) elements allowed past 2e-2 relative


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


def assert_float_close(got: np.ndarray, ref: np.ndarray, dtype: str, what: str,
                       per_element: bool = True) -> float:
    """per_element=False skips the share-of-significant-elements check: for FP8
    rows downstream of h's codes, where one code that moved by a step (reading of
    h's rounding boundary) perturbs every element of the row a little."""
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
    # the max-normalised bar alone would let an error confined to small values pass:
    # also the L2-relative error, and among the significant elements (|ref| above
    # the tensor's rms) the share whose own relative error exceeds the bar
    nr = float(np.linalg.norm(r))
    if nr > 0:
        l2 = float(np.linalg.norm(g - r)) / nr
        assert l2 <= BF16_REL_TOL, f"{what}: L2-relative error {l2:.3e}"
        big = np.abs(r) > np.sqrt(np.mean(r * r))
        if per_element and big.any():
            frac = float(np.mean(np.abs(g[big] - r[big]) > BF16_REL_TOL * np.abs(r[big])))
            assert frac <= SIGNIFICANT_FRAC, f"{what}: {frac:.2%} of the significant elements beyond the bar"
    return rel


def to_device(inp: MoEInputs, device="cuda") -> MoEInputs:
    mv = lambda t: None if t is None else t.to(device)
    return MoEInputs(logits=mv(inp.logits), bias=mv(inp.bias), x=mv(inp.x), w13=mv(inp.w13),
                     w2=mv(inp.w2), w13s=mv(inp.w13s), w2s=mv(inp.w2s))


def run_gpu_steps(wl: MoEWorkload, inp: MoEInputs, keep_rows: bool = True, fp8=None) -> dict:
    """Runs the six ABI steps chunk by chunk on the current CUDA stream.

    fp8: for a workload with ffn_fp8, the device (w13 codes, w13 scales, w2
    codes, w2 scales).  ffn_fp8 = 1: x is quantised once by rows, its codes are
    permuted and step 5 is moe_grouped_swiglu_ffn_fp8.  ffn_fp8 = 2: the
    permute quantises by 32-value blocks (moe_permute_quantize_fp8_blocks) and
    step 5 is moe_grouped_swiglu_ffn_mxfp8 (no bf16 h)."""
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
    xq = xs = None
    mx = wl.ffn_fp8 == 2
    if wl.ffn_fp8 and not mx:
        xq, xs = moe.quantize_fp8(inp.x)
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
        xr = torch.empty((max(nmax, 1), H), dtype=torch.uint8 if wl.ffn_fp8 else wl.torch_dtype,
                         device=dev)
        xsf = hsf = None
        if mx:
            xsf = torch.full((max(nmax, 1), H // 32), 7, dtype=torch.uint8, device=dev)
            moe.moe_permute_quantize_fp8_blocks(cfg, inp.x, pos, tb, tc, xr, xsf)
        else:
            moe.moe_permute(cfg, xq if wl.ffn_fp8 else inp.x, pos, tb, tc, xr)
        h = None if mx else torch.empty((max(nmax, 1), I), dtype=wl.torch_dtype, device=dev)
        y = None if wl.reduce_dense else torch.empty((max(nmax, 1), H), dtype=wl.torch_dtype, device=dev)
        hq = hsc = None
        if mx:
            hq = torch.empty((max(nmax, 1), I), dtype=torch.uint8, device=dev)
            hsf = torch.full((max(nmax, 1), I // 32), 7, dtype=torch.uint8, device=dev)
            w13q, w13s, w2q, w2s = fp8
            moe.moe_grouped_swiglu_ffn_mxfp8(cfg, nmax, xr, xsf, eoff, w13q, w13s, w2q, w2s, hq, hsf, y,
                                             rt, rs, topk_w, red, ws)
        elif wl.ffn_fp8:
            hq = torch.empty((max(nmax, 1), I), dtype=torch.uint8, device=dev)
            hsc = torch.empty((max(nmax, 1),), dtype=torch.uint8, device=dev)
            w13q, w13s, w2q, w2s = fp8
            moe.moe_grouped_swiglu_ffn_fp8(cfg, nmax, xr, xs, eoff, w13q, w13s, w2q, w2s, h, hq, hsc,
                                           y, rt, rs, topk_w, red, ws)
        else:
            moe.moe_grouped_swiglu_ffn(cfg, nmax, xr, eoff, inp.w13, inp.w2, h, y, rt, rs, topk_w,
                                       red, ws)
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
            ch.update(xr=storage_np(xr[:n]), h=None if h is None else storage_np(h[:n]),
                      xsf=None if xsf is None else xsf[:n].cpu().numpy(),
                      hsf=None if hsf is None else hsf[:n].cpu().numpy(),
                      y=None if y is None else storage_np(y[:n]),
                      ys=None if ys is None else storage_np(ys),
                      hq=None if hq is None else hq[:n].cpu().numpy(),
                      hs=None if hsc is None else hsc[:n].cpu().numpy())
        else:
            ch.update(xr_dev=xr, h_dev=h, y_dev=y, ys_dev=ys, hq_dev=hq, hs_dev=hsc, xsf_dev=xsf,
                      hsf_dev=hsf)
        chunks.append(ch)
    status = moe.moe_device_status(ws)
    torch.cuda.synchronize()
    return dict(topk_idx=topk_idx.cpu().numpy(), topk_w=topk_w.cpu().numpy(),
                counts=counts.cpu().numpy(), keep=keep.cpu().numpy(), kept_counts=kept.cpu().numpy(),
                chunks=chunks, out=out, status=status,
                xq=None if xq is None else xq.cpu().numpy(), xs=None if xs is None else xs.cpu().numpy())


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


def oracle_fp8_weights(inp: MoEInputs, experts=None) -> dict:
    """The oracle's E4M3 codes and UE8M0 row scales of the expert weights (all
    experts, or a dict for the listed ones): w13q [E, 2I, H], w13s [E, 2I],
    w2q [E, H, I], w2s [E, H]."""
    def q(w):
        a = storage_np(w)
        c, s = oracle.quantize_rows(a.reshape(-1, a.shape[-1]))
        return c.reshape(a.shape), s.reshape(a.shape[:-1])
    if experts is None:
        w13q, w13s = q(inp.w13)
        w2q, w2s = q(inp.w2)
        return dict(w13q=w13q, w13s=w13s, w2q=w2q, w2s=w2s)
    out = {}
    for e in experts:
        w13q, w13s = q(inp.w13[e])
        w2q, w2s = q(inp.w2[e])
        out[e] = dict(w13q=w13q, w13s=w13s, w2q=w2q, w2s=w2s)
    return out


def fp8_weights_to_device(wq: dict, device="cuda"):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
    return t(wq["w13q"]), t(wq["w13s"]), t(wq["w2q"]), t(wq["w2s"])


def oracle_fp8_ffn_and_out(wl: MoEWorkload, inp: MoEInputs, orc: dict, wq: dict):
    """The oracle's FP8 layer after routing: x quantised by rows, its codes
    permuted, the FP8 SwiGLU row by row, then the combine (decode form: over
    the unrounded y)."""
    x = storage_np(inp.x)
    xq, xs = oracle.quantize_rows(x)
    tc = wl.T // wl.n_chunks
    out = np.zeros((wl.T, wl.H), np.uint16)
    res = []
    for c, lay in enumerate(orc["layouts"]):
        n = lay["N"]
        xrq = oracle.permute(xq, lay["recv_token"])
        h = np.zeros((n, wl.I), np.uint16)
        hq = np.zeros((n, wl.I), np.uint8)
        hs = np.zeros(n, np.uint8)
        y = np.zeros((n, wl.H), np.uint16)
        ye = np.zeros((n, wl.H), np.float64)
        eoff = lay["expert_offsets"]
        for e in range(wl.E):
            for p in range(int(eoff[e]), int(eoff[e + 1])):
                h[p], hq[p], hs[p], y[p], ye[p] = oracle.ffn_row_fp8(
                    xrq[p], xs[lay["recv_token"][p]], wq["w13q"][e], wq["w13s"][e],
                    wq["w2q"][e], wq["w2s"][e])
        if wl.reduce_dense:
            oracle.combine_exact(ye, lay["pos"], orc["topk_w"], wl.T, np.uint16, c * tc, out)
        else:
            oracle.combine(y, lay["pos"], orc["topk_w"], wl.T, c * tc, out)
        res.append(dict(xrq=xrq, h=h, hq=hq, hs=hs, y=y))
    return dict(xq=xq, xs=xs, chunks=res, out=out)


def _signed_code(c):
    """E4M3 codes as signed integers ordered like their values (magnitude field
    with the sign), so that neighbouring representable values differ by one."""
    c = np.asarray(c, np.int32)
    return np.where(c & 0x80, -(c & 0x7F), c & 0x7F)


def assert_codes_close(got_codes, got_scales, ref_codes, ref_scales, what, min_equal=0.99):
    """Quantised rows whose inputs differ by float rounding (h summed in fp32 on the
    GPU, in fp64 by the oracle, then rounded to bf16): a value that sits on a
    rounding boundary can land one code away.  So: almost every code and scale
    equal; where the scales agree, every differing code is a neighbour of the
    oracle's (one E4M3 step); the dequantised rows of the other rows within the
    bf16 bar."""
    if ref_codes.size == 0:
        return
    assert (got_codes == ref_codes).mean() >= min_equal, f"{what}: codes differ too often"
    got_scales, ref_scales = np.asarray(got_scales), np.asarray(ref_scales)
    assert (got_scales == ref_scales).mean() >= min_equal, f"{what}: scales differ too often"
    same = (got_scales == ref_scales).reshape(-1)
    g2 = np.asarray(got_codes).reshape(len(same), -1)
    r2 = np.asarray(ref_codes).reshape(len(same), -1)
    step = np.abs(_signed_code(g2[same]) - _signed_code(r2[same]))
    assert step.size == 0 or step.max() <= 1, f"{what}: a code differs by {step.max()} steps"
    if (~same).any():
        assert_float_close(oracle.dequantize_rows(g2[~same], got_scales.reshape(-1)[~same]),
                           oracle.dequantize_rows(r2[~same], ref_scales.reshape(-1)[~same]), "bf16", what)
