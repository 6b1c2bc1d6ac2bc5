#!/usr/bin/env python
"""Benchmark of the expert-parallel MoE layer hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

One step = one pass of the whole layer (router top-k, capacity clip, dispatch
layout, permute, grouped SwiGLU FFN, combine) over one batch of seeded
synthetic inputs that are resident in HBM.  The default workload is the
largest single-GPU configuration, the DeepSeek-V3-shaped prefill layer
(T=8192, H=7168, E=256, k=8, I=2048, bf16, EP=8 logical ranks, two dispatch
chunks pipelined on two streams).

Prints one JSON line (rank 0).  Besides the contract keys it reports a
per-stage breakdown, dispatch+combine HBM GB/s, FFN TFLOP/s, the roofline of
the dominant kernel (the grouped FFN), an end-to-end number through the
public API with host buffers, and the CPU oracle timed on a bounded sample.
For a chunked workload the same line also carries the FFN's roofline with one
chunk (``roofline_unchunked``: every expert's weights read once per layer pass)
and ``overlap``: the two-stream step against the same kernels on one stream.

With --gpus N > 1 (launched by torchrun) every rank runs an independent
replica of the workload (the layer's EP ranks are logical, inside one GPU),
so there is no data-path collective; the time is the max over ranks and the
value counts the tokens of all ranks (weak scaling).

--impl reference times the CPU oracle (plain C, one core) on the same
workload, each step the whole layer over a sub-batch of its first tokens (a
multiple of the logical EP size), and prints the same line with
"impl": "reference".
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/sec at 1 B200; dispatch+combine HBM GB/s; FFN tensor-pipe %"
UNIT = "tokens/s"
L2_FLUSH_BYTES = 512 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic of the grouped FFN (both GEMM launches) per layer pass, from one
# ncu capture (dram__bytes_read.sum + dram__bytes_write.sum); see
# profiles/ffn_tcgen05_qwen3_30b_a3b.md.  Keyed by workload; ``src`` is the
# sha256 prefix of the kernel source the counters were taken on - a changed
# kernel reports null until it is captured again.
FFN_TRAFFIC = {
    "qwen3_30b_a3b": {"bytes": (942.794240 + 45.979648 + 453.990656 + 113.344512) * 1e6,
                      "src": "52e786192f9b24d0"},
    # both GEMM launches and the quantisation of h between them
    "qwen3_30b_a3b_fp8": {"bytes": (471.297792 + 42.182400 + 50.341376 + 1.413888 + 226.896384 +
                                    96.848640) * 1e6, "src": "18a4e475b021b023"},
    "qwen3_30b_a3b_mxfp8": {"bytes": (484.897024 + 24.313600 + 233.751296 + 105.241344) * 1e6,
                            "src": "f91c44b09b122286"},
    # captured with 32 of the 256 experts and 1024 tokens (the same 128 rows per
    # expert and chunk), scaled by 8 per chunk, two chunks; see
    # profiles/ffn_tcgen05_dsv3_prefill.md and profiles/ffn_mx_tcgen05_dsv3_prefill_mxfp8.md
    "dsv3_prefill": {"bytes": 2 * 8 * (1956.903168e6 + 18.358016e6 + 958.769664e6 + 54.941440e6),
                     "src": "52e786192f9b24d0", "chunks": 2},
    "dsv3_prefill_mxfp8": {"bytes": 2 * 8 * (1008.328192e6 + 11.598080e6 + 494.208000e6 + 49.762304e6),
                           "src": "f91c44b09b122286", "chunks": 2},
}


def workload_of(args):
    """The named workload, with the chunk count, token count or expert count
    overridden when asked (a smaller case of the same shape, e.g. for a
    counter capture); an overridden workload carries the changes in its name."""
    from combine_moe_route_12_b200.workload import WORKLOADS
    wl = WORKLOADS[args.config]
    over = {}
    if args.chunks is not None:
        over["n_chunks"] = args.chunks
    if getattr(args, "tokens", None) is not None:
        over["T"] = args.tokens
    if getattr(args, "experts", None) is not None:
        over["E"] = args.experts
    if not over:
        return wl
    tag = ",".join(f"{k}={v}" for k, v in over.items())
    return wl.with_(name=f"{wl.name}[{tag}]", **over)


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--config", default="dsv3_prefill")
    p.add_argument("--chunks", type=int, default=None,
                   help="override the workload's dispatch chunk count (e.g. 1 for the unchunked DSV3 prefill FFN)")
    p.add_argument("--tokens", type=int, default=None, help="override the workload's token count T")
    p.add_argument("--experts", type=int, default=None, help="override the workload's expert count E")
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true", help="skip the CPU oracle sample")
    p.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end pass")
    p.add_argument("--no-unchunked", action="store_true",
                   help="skip the one-chunk FFN breakdown of a chunked workload")
    p.add_argument("--no-overlap", action="store_true",
                   help="skip the one-stream replay of a chunked workload")
    p.add_argument("--backward", action="store_true",
                   help="also time the backward: the layer's backward with the dispatch outputs saved "
                        "and recomputed, the expert FFN's backward step (with its roofline), and the "
                        "row passes on the last chunk (backward and backward_row_passes objects)")
    p.add_argument("--seed", type=int, default=None)
    p.add_argument("--no-graph", action="store_true",
                   help="time eager launches instead of replaying a captured CUDA graph of the layer")
    return p.parse_args(argv)


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank scalar over the process group (identity without one).
    NCCL needs a CUDA tensor; gloo (used by the CPU tests) a CPU one."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    if device is None:
        device = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_src_hash(fp8: bool = False, mx: bool = False):
    """Hash of the FFN's sources: the grouped GEMM kernel, and for the FP8 FFN also
    the row quantisation between its launches (the block-scaled FP8 FFN: its own
    kernel).  Recorded traffic holds only for these bytes."""
    h = hashlib.sha256()
    names = (("ffn_mx_tcgen05.cu", "ffn_pair.cuh") if mx else
             ("ffn_tcgen05.cu", "ffn_pair.cuh", "fp8_quant.cu") if fp8 else ("ffn_tcgen05.cu", "ffn_pair.cuh"))
    for name in names:
        with open(os.path.join(ROOT, "combine_moe_route_12_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML (reads
    only) on a background thread while the GPU is busy."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples = []
        self.max_mhz = None
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - depends on the NVML of the machine
            self.err = str(e)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                pw = nv.nvmlDeviceGetPowerUsage(self._h) / 1000.0
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                except Exception:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
                util = nv.nvmlDeviceGetUtilizationRates(self._h).gpu
                self.samples.append((sm, pw, rs, util))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread:
            self._stop.set()
            self._thread.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "note": "no NVML samples"}
        busy = [s for s in self.samples if s[3] > 0] or self.samples
        reasons = set()
        for s in busy:
            for name, bit in self.REASONS.items():
                if s[2] & bit and name != "gpu_idle":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s[0] for s in busy), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(busy),
                "power_w_max": max(s[1] for s in busy)}


# --------------------------------------------------------------------------- workload

def kernels_per_step(wl) -> int:
    # route 1; clip 1 without a capacity (one pass), 2 with capacity 0 (prep, mark),
    # 4 with a positive capacity (+ gather, select);
    # per chunk: layout 2 (hist, scatter), permute 1, FFN 2 (two GEMM launches),
    # combine or finalize 1
    # with a shared expert, per chunk 3 more (its offsets and two GEMM launches);
    # with the FP8 FFN, per chunk 1 more (h's row quantisation), 2 when x's
    # quantisation is not fused into the permute (H > 8192)
    # with the block-scaled FP8 FFN (ffn_fp8 = 2) nothing more: x is quantised inside
    # the permute and h inside GEMM1
    clip = 4 if wl.capacity > 0 else 2 if wl.capacity == 0 else 1
    fp8 = 0 if is_mx(wl) else (1 if fused_permute_quant(wl) else 2) if wl.ffn_fp8 else 0
    return 1 + clip + wl.n_chunks * (6 + (3 if wl.shared_I > 0 else 0) + fp8)


def fused_permute_quant(wl) -> bool:
    """The FP8 path quantises x inside the permute for rows of up to 8192 values."""
    return bool(wl.ffn_fp8) and wl.H <= 8192


def is_mx(wl) -> bool:
    """The FP8 FFN with one UE8M0 scale per 32 K values (ffn_fp8 = 2)."""
    return wl.ffn_fp8 == 2


def algorithmic(wl, n_kept_chunks, active_chunks, tokens_read=None):
    """Bytes / flops the method must move or compute (nothing for dropped rows;
    the permute reads the x rows of the tokens_read tokens that keep at least one
    slot, all T when not given).

    ffn_bytes: per layer pass, the weights of every expert with a row in each
    chunk (each chunk streams them once), the receive rows read by GEMM1, h
    written and read back, and y written (decode form: the dense fp32 buffer
    read and written once instead).

    FP8 FFN: weights and receive rows are one-byte codes (plus one scale byte
    per weight row); h is written in bf16, read by its quantisation, whose
    codes are written and read by GEMM2; the permute stage reads the kept
    tokens' bf16 rows and writes their codes (H <= 8192: one fused pass), or
    quantises all of x, writes its codes and permutes them (longer rows).
    Block-scaled FP8 (ffn_fp8 = 2): one scale byte per 32 values beside every
    code row (weights, receive rows, h); h is quantised inside GEMM1, so only
    its codes and scales are written and read."""
    b = wl.elem_bytes
    N = sum(n_kept_chunks)
    tok_bytes = wl.T * wl.H * b
    read_bytes = (wl.T if tokens_read is None else tokens_read) * wl.H
    y_bytes = N * wl.H * b
    out_bytes = 2 * wl.T * wl.H * 4 if wl.reduce_dense else y_bytes
    if is_mx(wl):
        row_bytes = N * wl.H * 33 // 32
        w_bytes = sum(active_chunks) * 3 * wl.H * wl.I * 33 // 32
        permute_bytes = read_bytes * b + row_bytes
        h_bytes = 2 * N * wl.I * 33 // 32
    elif wl.ffn_fp8:
        row_bytes = N * wl.H
        w_bytes = sum(active_chunks) * (3 * wl.H * wl.I + 2 * wl.I + wl.H)
        if fused_permute_quant(wl):
            permute_bytes = read_bytes * b + row_bytes
        else:
            permute_bytes = tok_bytes + wl.T * wl.H + read_bytes + row_bytes
        h_bytes = N * wl.I * (2 * b + 2)
    else:
        row_bytes = y_bytes
        w_bytes = sum(active_chunks) * 3 * wl.H * wl.I * b
        permute_bytes = read_bytes * b + row_bytes
        h_bytes = 2 * N * wl.I * b
    return {
        "permute_bytes": permute_bytes,
        "combine_bytes": (0 if wl.reduce_dense else y_bytes) + tok_bytes,
        "ffn_flops": 6.0 * wl.H * wl.I * N,
        "ffn_bytes": w_bytes + row_bytes + h_bytes + out_bytes,
        "N": N,
    }


class StepBuffers:
    """Every buffer the six ABI calls of one unchunked step touch."""

    def __init__(self, moe, wl, cfg, dev):
        import torch
        T, E, k, H, I, ep = wl.T, wl.E, wl.k, wl.H, wl.I, wl.ep
        self.ws = moe.alloc_workspace(moe.workspace_bytes(cfg), dev)
        self.topk_idx = torch.empty(T, k, dtype=torch.int32, device=dev)
        self.topk_w = torch.empty(T, k, dtype=torch.float32, device=dev)
        self.counts = torch.empty(E, dtype=torch.int32, device=dev)
        self.keep = torch.empty(T, k, dtype=torch.uint8, device=dev)
        self.kept = torch.empty(E, dtype=torch.int32, device=dev)
        tc = T // wl.n_chunks
        self.tc = tc
        self.nmax = moe.max_recv_rows(cfg, tc)
        n = max(self.nmax, 1)
        self.eoff = torch.empty(E + 1, dtype=torch.int32, device=dev)
        self.roff = torch.empty(ep + 1, dtype=torch.int32, device=dev)
        self.rt = torch.empty(n, dtype=torch.int32, device=dev)
        self.rs = torch.empty(n, dtype=torch.int32, device=dev)
        self.pos = torch.empty(tc, k, dtype=torch.int32, device=dev)
        self.spl = torch.empty(ep, ep, dtype=torch.int32, device=dev)
        self.xr = torch.empty(n, H, dtype=torch.uint8 if wl.ffn_fp8 else wl.torch_dtype, device=dev)
        if is_mx(wl):
            self.xsf = torch.empty(n, H // 32, dtype=torch.uint8, device=dev)
            self.hq = torch.empty(n, I, dtype=torch.uint8, device=dev)
            self.hsf = torch.empty(n, I // 32, dtype=torch.uint8, device=dev)
        elif wl.ffn_fp8:
            self.xq = torch.empty(T, H, dtype=torch.uint8, device=dev)
            self.xsc = torch.empty(T, dtype=torch.uint8, device=dev)
            self.hq = torch.empty(n, I, dtype=torch.uint8, device=dev)
            self.hsc = torch.empty(n, dtype=torch.uint8, device=dev)
        self.h = torch.empty(n, I, dtype=wl.torch_dtype, device=dev)
        self.y = None if wl.reduce_dense else torch.empty(n, H, dtype=wl.torch_dtype, device=dev)
        self.red = torch.zeros(T, H, dtype=torch.float32, device=dev) if wl.reduce_dense else None
        self.out = torch.empty(T, H, dtype=wl.torch_dtype, device=dev)
        self.hs = self.ys = None
        if wl.shared_I > 0:
            self.hs = torch.empty(tc, wl.shared_I, dtype=wl.torch_dtype, device=dev)
            self.ys = torch.empty(tc, H, dtype=wl.torch_dtype, device=dev)


def n_marks(wl) -> int:
    return 3 + 5 * wl.n_chunks


def run_steps(moe, wl, cfg, inp, B, ev=None, fp8=None):
    """One layer pass through the step ABI on the current stream.  ev: list of
    n_marks(wl) events recorded between the stages, or None.  fp8: the device
    (w13 codes, w13 scales, w2 codes, w2 scales) of an FP8 workload; its
    permute stage quantises the chunk's x rows (inside the permute for H <= 8192)."""
    rec = (lambda i: ev[i].record()) if ev is not None else (lambda i: None)
    rec(0)
    moe.moe_route_topk(cfg, inp.logits, inp.bias, B.topk_idx, B.topk_w, B.counts, B.ws)
    rec(1)
    moe.moe_capacity_clip(cfg, B.topk_idx, B.topk_w, B.counts, B.keep, B.kept, B.ws)
    if wl.reduce_dense:
        B.red.zero_()
    rec(2)
    for c in range(wl.n_chunks):
        tb = c * B.tc
        base = 3 + 5 * c
        moe.moe_dispatch_layout(cfg, tb, B.tc, B.topk_idx, B.keep, B.eoff, B.roff, B.rt, B.rs,
                                B.pos, B.spl, None, B.ws)
        rec(base)
        if is_mx(wl):
            moe.moe_permute_quantize_fp8_blocks(cfg, inp.x, B.pos, tb, B.tc, B.xr, B.xsf)
        elif fused_permute_quant(wl):
            moe.moe_permute_quantize_fp8(cfg, inp.x, B.pos, tb, B.tc, B.xr, B.xsc)
        elif wl.ffn_fp8:
            moe.moe_quantize_fp8_rows(inp.x[tb:tb + B.tc], B.xq[tb:tb + B.tc], B.xsc[tb:tb + B.tc])
            moe.moe_permute(cfg, B.xq, B.pos, tb, B.tc, B.xr)
        else:
            moe.moe_permute(cfg, inp.x, B.pos, tb, B.tc, B.xr)
        rec(base + 1)
        if is_mx(wl):
            w13q, w13s, w2q, w2s = fp8
            moe.moe_grouped_swiglu_ffn_mxfp8(cfg, B.nmax, B.xr, B.xsf, B.eoff, w13q, w13s, w2q, w2s, B.hq,
                                             B.hsf, B.y, B.rt, B.rs, B.topk_w, B.red, B.ws)
        elif wl.ffn_fp8:
            w13q, w13s, w2q, w2s = fp8
            moe.moe_grouped_swiglu_ffn_fp8(cfg, B.nmax, B.xr, B.xsc, B.eoff, w13q, w13s, w2q, w2s,
                                           B.h, B.hq, B.hsc, B.y, B.rt, B.rs, B.topk_w, B.red, B.ws)
        else:
            moe.moe_grouped_swiglu_ffn(cfg, B.nmax, B.xr, B.eoff, inp.w13, inp.w2, B.h, B.y, B.rt,
                                       B.rs, B.topk_w, B.red, B.ws)
        rec(base + 2)
        if wl.shared_I > 0:
            moe.moe_shared_expert_ffn(cfg, tb, B.tc, inp.x, inp.w13s, inp.w2s, B.hs, B.ys, B.ws)
        rec(base + 3)
        if wl.reduce_dense:
            moe.moe_reduce_finalize(cfg, B.red, tb, B.tc, B.out, y_shared=B.ys)
        else:
            moe.moe_combine(cfg, B.y, B.pos, B.topk_w, tb, B.tc, B.out, y_shared=B.ys)
        rec(base + 4)


def backward_row_passes(moe, wl, cfg, B, n_rows, peaks, flush, args):
    """Times the backward's row passes on the last chunk's layout (B holds it after
    the breakdown pass): the combine's backward against the forward's y rows, the
    permute's backward of synthetic receive-row gradients, and the routing's
    backward of the resulting dw over all T tokens.  HBM bytes per pass: combine
    tc·H·b (dout) + 2·N·H·b (y read, dy written) + 4·tc·k (dw); permute N·H·b +
    tc·H·b; routing 4·T·E written (+ 12·T·k read)."""
    import torch
    dev = B.xr.device
    T, H, k, E, tc = wl.T, wl.H, wl.k, wl.E, B.tc
    tb = (wl.n_chunks - 1) * tc
    b = wl.elem_bytes
    g = torch.Generator(device=dev).manual_seed(17)
    dout = torch.randn(T, H, generator=g, device=dev).to(wl.torch_dtype)
    dxr = torch.randn(max(B.nmax, 1), H, generator=g, device=dev).to(wl.torch_dtype)
    dy = torch.empty(max(B.nmax, 1), H, dtype=wl.torch_dtype, device=dev)
    dx = torch.empty(T, H, dtype=wl.torch_dtype, device=dev)
    dw = torch.zeros(T, k, dtype=torch.float32, device=dev)
    dl = torch.empty(T, E, dtype=torch.float32, device=dev)
    db = torch.empty(E, dtype=torch.float32, device=dev)
    t = {"combine": 0.0, "permute": 0.0, "route": 0.0}
    for i in range(args.warmup + args.steps):
        flush.fill_(1)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        ev[0].record()
        moe.moe_combine_backward(cfg, dout, B.y, B.pos, B.topk_w, tb, tc, dy, dw)
        ev[1].record()
        moe.moe_permute_backward(cfg, dxr, B.pos, tb, tc, dx)
        ev[2].record()
        moe.moe_route_backward(cfg, B.topk_idx, B.topk_w, dw, dl, db, B.ws)
        ev[3].record()
        torch.cuda.synchronize()
        if i >= args.warmup:
            for j, name in enumerate(("combine", "permute", "route")):
                t[name] += ev[j].elapsed_time(ev[j + 1]) / args.steps
    if moe.moe_device_status(B.ws) != 0:
        raise RuntimeError("device status bits set during the backward passes")
    cb = tc * H * b + 2 * n_rows * H * b + 4 * tc * k
    pb = n_rows * H * b + tc * H * b
    rb = 4 * T * E + 12 * T * k
    gbs = lambda by, ms: by / (ms * 1e-3) / 1e9 if ms > 0 else None
    return {"chunk_tokens": tc, "rows": n_rows,
            "combine_bwd": {"ms": round(t["combine"], 4), "gbs": gbs(cb, t["combine"]),
                            "frac": gbs(cb, t["combine"]) / peaks["hbm_gbs"] if t["combine"] > 0 else None},
            "permute_bwd": {"ms": round(t["permute"], 4), "gbs": gbs(pb, t["permute"]),
                            "frac": gbs(pb, t["permute"]) / peaks["hbm_gbs"] if t["permute"] > 0 else None},
            "route_bwd": {"ms": round(t["route"], 4), "gbs": gbs(rb, t["route"])},
            "timing": "CUDA events around each eager launch, L2 flushed before each pass triple"}


def ffn_backward_algorithmic(wl, N, active):
    """Bytes and flops of the expert FFN's backward over N receive rows with
    `active` experts holding rows: W13 read twice (g | u recomputed; dxr) and W2
    once (dh); xr and dy read twice (data and weight gradients); g | u written
    and read; h written and read; dg | du written and read twice; dxr written;
    the fp32 weight gradients of all E experts written once.  Flops:
    2 * N * (2IH + HI + 2IH + HI + 2IH) = 16 * H * I * N."""
    b = wl.elem_bytes
    H, I = wl.H, wl.I
    w = 5 * active * H * I * b
    act = N * (2 * H + 2 * H + 2 * 2 * I + 2 * I + 3 * 2 * I + H) * b
    dw = wl.E * 3 * H * I * 4
    return {"bytes": w + act + dw, "flops": 16.0 * H * I * N, "weight_bytes": w, "act_bytes": act,
            "dw_bytes": dw}


def layer_backward(moe, wl, cfg, inp, layer, flush, args, peaks, peak_src):
    """Times the layer's backward (moe_layer_backward) with the dispatch outputs
    saved by the forward and with them recomputed, alternating step by step,
    and the expert FFN's backward step alone over the whole batch's receive rows
    (one-chunk layout), with its roofline."""
    import torch
    dev = inp.x.device
    T, H, E, k, I = wl.T, wl.H, wl.E, wl.k, wl.I
    dt = wl.torch_dtype
    nmax = moe.max_recv_rows(cfg, T // wl.n_chunks)
    xr_s = torch.empty(wl.n_chunks, max(nmax, 1), H, dtype=dt, device=dev)
    y_s = torch.empty(wl.n_chunks, max(nmax, 1), H, dtype=dt, device=dev)
    out = torch.empty(T, H, dtype=dt, device=dev)
    s = torch.cuda.current_stream()
    moe.moe_forward_chunked_save(cfg, inp.logits, inp.bias, inp.x, inp.w13, inp.w2, out, layer.topk_idx,
                                 layer.topk_w, layer.keep, None, xr_s, y_s, layer.ws, s, s, inp.w13s, inp.w2s)
    g = torch.Generator(device=dev).manual_seed(17)
    dout = torch.randn(T, H, generator=g, device=dev).to(dt)
    bws = moe.alloc_workspace(moe.backward_workspace_bytes(cfg), dev)
    dx = torch.empty(T, H, dtype=dt, device=dev)
    dl = torch.empty(T, E, dtype=torch.float32, device=dev)
    db = torch.empty(E, dtype=torch.float32, device=dev)
    dw13 = torch.empty(E, 2 * I, H, dtype=torch.float32, device=dev)
    dw2 = torch.empty(E, H, I, dtype=torch.float32, device=dev)
    sh = {}
    if wl.shared_I > 0:
        sh = dict(w13_shared=inp.w13s, w2_shared=inp.w2s,
                  dw13_shared=torch.empty(2 * wl.shared_I, H, device=dev),
                  dw2_shared=torch.empty(H, wl.shared_I, device=dev))

    def bwd(saved):
        moe.moe_layer_backward(cfg, inp.x, dout, inp.w13, inp.w2, layer.topk_idx, layer.topk_w, layer.keep,
                               dx, dl, db, dw13, dw2, bws, xr_saved=xr_s if saved else None,
                               y_saved=y_s if saved else None, **sh)

    for _ in range(max(1, args.warmup)):
        bwd(True)
        bwd(False)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for i in range(args.steps):
        flush.fill_(1)
        ev[i][0].record()
        bwd(True)
        ev[i][1].record()
        flush.fill_(1)
        ev[i][2].record()
        bwd(False)
        ev[i][3].record()
    torch.cuda.synchronize()
    if moe.moe_device_status(bws) != 0:
        raise RuntimeError("device status bits set during the layer backward")
    save_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / args.steps
    rec_ms = sum(e[2].elapsed_time(e[3]) for e in ev) / args.steps
    del bws, xr_s, y_s

    # the expert FFN's backward step over the whole batch in one receive buffer
    w1 = wl.with_(n_chunks=1)
    c1 = moe.config_from_workload(w1)
    ws1 = moe.alloc_workspace(moe.workspace_bytes(c1), dev)
    n1 = moe.max_recv_rows(c1, T)
    eoff = torch.empty(E + 1, dtype=torch.int32, device=dev)
    roff = torch.empty(w1.ep + 1, dtype=torch.int32, device=dev)
    rt = torch.empty(max(n1, 1), dtype=torch.int32, device=dev)
    rs = torch.empty(max(n1, 1), dtype=torch.int32, device=dev)
    pos = torch.empty(T, k, dtype=torch.int32, device=dev)
    spl = torch.empty(w1.ep, w1.ep, dtype=torch.int32, device=dev)
    moe.moe_dispatch_layout(c1, 0, T, layer.topk_idx, layer.keep, eoff, roff, rt, rs, pos, spl, None, ws1)
    xr = torch.empty(max(n1, 1), H, dtype=dt, device=dev)
    moe.moe_permute(c1, inp.x, pos, 0, T, xr)
    dyr = torch.randn(max(n1, 1), H, generator=g, device=dev).to(dt)
    gu = torch.empty(max(n1, 1), 2 * I, dtype=dt, device=dev)
    hh = torch.empty(max(n1, 1), I, dtype=dt, device=dev)
    dgu = torch.empty(max(n1, 1), 2 * I, dtype=dt, device=dev)
    dxr = torch.empty(max(n1, 1), H, dtype=dt, device=dev)
    torch.cuda.synchronize()
    N = int(eoff[E].item())
    active = int(((eoff[1:] - eoff[:-1]) > 0).sum().item())

    def step():
        moe.moe_grouped_swiglu_ffn_backward(c1, n1, xr, dyr, eoff, inp.w13, inp.w2, gu, hh, dgu, dxr,
                                            dw13, dw2, 0, ws1)

    for _ in range(max(1, args.warmup)):
        step()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for i in range(args.steps):
        flush.fill_(1)
        evs[i][0].record()
        step()
        evs[i][1].record()
    torch.cuda.synchronize()
    if moe.moe_device_status(ws1) != 0:
        raise RuntimeError("device status bits set during the FFN backward")
    ffn_ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
    alg = ffn_backward_algorithmic(wl, N, active)
    t = ffn_ms / 1e3
    tflops = alg["flops"] / t / 1e12
    gbs = alg["bytes"] / t / 1e9
    t_flop = alg["flops"] / (peaks["bf16_tflops"] * 1e12)
    t_byte = alg["bytes"] / (peaks["hbm_gbs"] * 1e9)
    hbm = t_byte > t_flop
    return {
        "layer_backward_ms": {"save_dispatch": round(save_ms, 4), "recompute": round(rec_ms, 4),
                              "recompute_minus_save": round(rec_ms - save_ms, 4),
                              "tokens_per_s_save": T / (save_ms / 1e3),
                              "timing": "moe_layer_backward, the two modes alternated step by step, "
                                        "L2 flushed before each"},
        "ffn_backward": {"kernel": "moe_grouped_swiglu_ffn_backward: g|u, dh + SwiGLU backward, dxr "
                                   "(ffn_gemm_tcgen05_kernel), dW2 and dW13 (wgrad_tcgen05_kernel)",
                         "rows": N, "active_experts": active, "ms": round(ffn_ms, 4),
                         "bound": "hbm" if hbm else "tensor",
                         "achieved": gbs if hbm else tflops,
                         "peak": peaks["hbm_gbs"] if hbm else peaks["bf16_tflops"],
                         "unit": "GB/s" if hbm else "TFLOP/s",
                         "frac": gbs / peaks["hbm_gbs"] if hbm else tflops / peaks["bf16_tflops"],
                         "tflops": tflops, "gbs": gbs,
                         "tensor_frac": tflops / peaks["bf16_tflops"],
                         "tensor_frac_sustained": tflops / peaks["bf16_tflops_sustained"],
                         "hbm_frac": gbs / peaks["hbm_gbs"],
                         "algorithmic": alg, "peak_source": peak_src},
    }


def stage_times(wl, ev, per_chunk=False):
    """Per-stage milliseconds of one step recorded by run_steps (and, with
    per_chunk, the list of each chunk's dispatch_layout + permute time)."""
    t = {"route_topk": ev[0].elapsed_time(ev[1]), "capacity_clip": ev[1].elapsed_time(ev[2]),
         "dispatch_layout": 0.0, "permute": 0.0, "grouped_ffn": 0.0, "shared_expert": 0.0,
         "combine": 0.0}
    disp = []
    for c in range(wl.n_chunks):
        b = 3 + 5 * c
        prev = ev[2] if c == 0 else ev[b - 1]
        lay = prev.elapsed_time(ev[b])
        per = ev[b].elapsed_time(ev[b + 1])
        t["dispatch_layout"] += lay
        t["permute"] += per
        t["grouped_ffn"] += ev[b + 1].elapsed_time(ev[b + 2])
        t["shared_expert"] += ev[b + 2].elapsed_time(ev[b + 3])
        t["combine"] += ev[b + 3].elapsed_time(ev[b + 4])
        disp.append(lay + per)
    return (t, disp) if per_chunk else t


STAGES = ["route_topk", "capacity_clip", "dispatch_layout", "permute", "grouped_ffn",
          "shared_expert", "combine"]


def breakdown(moe, wl, cfg, inp, B, fp8, steps, flush, use_graph):
    """The step ABI on one stream with events between the stages, captured into a
    CUDA graph with the events (no host launch gaps; eager launches if capture
    fails), replayed `steps` times with the L2 flushed before each.  Returns
    (mean stage ms, mean per-chunk dispatch ms, mean step ms, mode)."""
    import torch
    mk = lambda: [torch.cuda.Event(enable_timing=True) for _ in range(n_marks(wl))]
    for _ in range(2):
        run_steps(moe, wl, cfg, inp, B, None, fp8)
    torch.cuda.synchronize()
    stage_ms = {s: 0.0 for s in STAGES}
    disp_ms = [0.0] * wl.n_chunks
    step_sum = 0.0
    bd_ev = mk()
    bd_graph = None
    if use_graph:
        try:
            # external events stay timing events inside a captured graph
            gev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(n_marks(wl))]
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                run_steps(moe, wl, cfg, inp, B, gev, fp8)
            torch.cuda.synchronize()
            g.replay()
            torch.cuda.synchronize()
            stage_times(wl, gev)          # raises if the events cannot be timed
            bd_graph, bd_ev = g, gev
        except Exception:
            bd_graph = None
            torch.cuda.synchronize()
    for _ in range(steps):
        flush.fill_(1)
        if bd_graph is not None:
            bd_graph.replay()
        else:
            run_steps(moe, wl, cfg, inp, B, bd_ev, fp8)
        torch.cuda.synchronize()
        st, dp = stage_times(wl, bd_ev, per_chunk=True)
        for s_, v in st.items():
            stage_ms[s_] += v / steps
        for c, v in enumerate(dp):
            disp_ms[c] += v / steps
        step_sum += bd_ev[0].elapsed_time(bd_ev[-1]) / steps
    if moe.moe_device_status(B.ws) != 0:
        raise RuntimeError("device status bits set during the breakdown pass")
    mode = "graph" if bd_graph is not None else "eager"
    del bd_graph
    return stage_ms, disp_ms, step_sum, mode


def index_path_ms(moe, wl, cfg, inp, B, steps, flush):
    """The index path (route, clip and the first chunk's dispatch layout) as one
    CUDA graph with no events inside, replayed `steps` times with the L2 flushed
    before each: milliseconds per replay, or None if capture fails.  The
    per-stage breakdown's events sit between graph nodes and add their own
    cost to every stage."""
    import torch

    def path():
        moe.moe_route_topk(cfg, inp.logits, inp.bias, B.topk_idx, B.topk_w, B.counts, B.ws)
        moe.moe_capacity_clip(cfg, B.topk_idx, B.topk_w, B.counts, B.keep, B.kept, B.ws)
        moe.moe_dispatch_layout(cfg, 0, B.tc, B.topk_idx, B.keep, B.eoff, B.roff, B.rt, B.rs, B.pos, B.spl,
                                None, B.ws)

    path()
    torch.cuda.synchronize()
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            path()
        torch.cuda.synchronize()
    except Exception:
        torch.cuda.synchronize()
        return None
    for _ in range(3):
        g.replay()
    total = 0.0
    for _ in range(steps):
        flush.fill_(1)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        total += a.elapsed_time(b)
    del g
    if moe.moe_device_status(B.ws) != 0:
        raise RuntimeError("device status bits set during the index path timing")
    return total / steps


def layout_counts(moe, wl, cfg, B):
    """Kept rows and active experts of each chunk, and the tokens with a kept slot."""
    n_kept, n_active = [], []
    for c in range(wl.n_chunks):
        moe.moe_dispatch_layout(cfg, c * B.tc, B.tc, B.topk_idx, B.keep, B.eoff, B.roff, B.rt, B.rs,
                                B.pos, B.spl, None, B.ws)
        n_kept.append(int(B.eoff[wl.E].item()))
        n_active.append(int(((B.eoff[1:] - B.eoff[:-1]) > 0).sum().item()))
    tokens_read = int((B.keep.view(wl.T, wl.k) != 0).any(dim=1).sum().item())
    return n_kept, n_active, tokens_read


def ffn_roofline(wl, alg, ffn_ms, peaks, peak_src, traffic):
    """The grouped FFN's roofline for one layer pass: its algorithmic bytes and
    flops over the measured duration, against the binding roof (HBM when the
    pass's flop per byte is below the ridge).  The tensor fraction is also given
    against the sustained bf16 figure (a long step runs under the power cap)."""
    ffn_s = ffn_ms / 1e3
    f8 = 2.0 if wl.ffn_fp8 else 1.0
    # the tensor peak of the FFN's operand type: the measured bf16 figure, times
    # the nominal dense FP8 / bf16 ratio (4.5 / 2.25) for E4M3 operands
    t_peak = peaks["bf16_tflops"] * f8
    t_peak_sus = peaks["bf16_tflops_sustained"] * f8
    t_peak_src = "bf16_tflops (burst) x 2 (nominal e4m3 / bf16)" if wl.ffn_fp8 else "bf16_tflops (burst)"
    t_flop = alg["ffn_flops"] / (t_peak * 1e12)
    t_byte = alg["ffn_bytes"] / (peaks["hbm_gbs"] * 1e9)
    hbm_bound = t_byte > t_flop
    tflops = alg["ffn_flops"] / ffn_s / 1e12 if ffn_s > 0 else None
    gbs = alg["ffn_bytes"] / ffn_s / 1e9 if ffn_s > 0 else None
    kname = ("grouped SwiGLU FFN (ffn_mx_tcgen05_kernel, GEMM1 with h quantised in its epilogue + GEMM2, "
             "E4M3 operands with one UE8M0 scale per 32 K values)") if is_mx(wl) else \
        ("grouped SwiGLU FFN (ffn_gemm_tcgen05_kernel, GEMM1 + GEMM2 per layer pass"
         + (", E4M3 operands, h quantised between them)" if wl.ffn_fp8 else ")"))
    return {"kernel": kname,
            "bound": "hbm" if hbm_bound else "tensor",
            "achieved": gbs if hbm_bound else tflops,
            "peak": peaks["hbm_gbs"] if hbm_bound else t_peak,
            "unit": "GB/s" if hbm_bound else "TFLOP/s",
            "frac": (gbs / peaks["hbm_gbs"] if hbm_bound else tflops / t_peak) if ffn_s > 0 else None,
            "traffic": traffic,
            "peak_source": f"{peak_src} " + ("hbm_gbs" if hbm_bound else t_peak_src),
            "algorithmic_per_launch": f"{alg['ffn_bytes']:.4g} B and 6*H*I*N = {alg['ffn_flops']:.4g} flop "
                                      f"over N={alg['N']} kept rows in {wl.n_chunks} chunk(s)",
            "ms": round(ffn_ms, 4),
            "tflops": tflops,
            "gbs": gbs,
            "tensor_frac": tflops / t_peak if tflops else None,
            "tensor_frac_sustained": tflops / t_peak_sus if tflops else None,
            "tensor_peak_sustained": t_peak_sus,
            "hbm_frac": gbs / peaks["hbm_gbs"] if gbs else None}


def dispatch_combine(alg, stage_ms, peaks, peak_src):
    dc_s = (stage_ms["permute"] + stage_ms["combine"]) / 1e3
    by = alg["permute_bytes"] + alg["combine_bytes"]
    gbs = by / dc_s / 1e9 if dc_s > 0 else None
    return {"achieved_gbs": gbs, "peak_gbs": peaks["hbm_gbs"],
            "frac": gbs / peaks["hbm_gbs"] if gbs else None, "bytes_per_step": by,
            "ms": round(stage_ms["permute"] + stage_ms["combine"], 4),
            "peak_source": f"{peak_src} hbm_gbs"}


# --------------------------------------------------------------------------- CPU oracle sample

def host_threads():
    """The host cores this process may run on (its affinity set)."""
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return max(1, os.cpu_count() or 1)


def oracle_rows(row_fn, rows_by_expert, threads):
    """Runs the oracle's FFN row `row_fn(p, e)` for every (expert, rows) item, the
    experts spread over `threads` host threads (the oracle's C calls release the
    interpreter lock; each row writes only its own outputs)."""
    import concurrent.futures as cf

    def work(item):
        e, ps = item
        for p in ps:
            row_fn(p, e)
    items = [(e, ps) for e, ps in rows_by_expert.items() if ps]
    if threads <= 1:
        for it in items:
            work(it)
        return
    with cf.ThreadPoolExecutor(threads) as ex:
        list(ex.map(work, items))


def oracle_sample(wl, logits, bias, x_np, fetch_expert, sample_tokens, shared=None, threads=1):
    """Times the oracle, as it stands, on a bounded sample: route + clip +
    layout + permute over all T tokens, then FFN + combine (+ the shared expert,
    `shared` = its host weights) for the rows of the first `sample_tokens`
    tokens, the FFN rows spread over `threads` host threads.  Returns (tokens/s
    extrapolated to the whole layer, seconds of wall time, description)."""
    import numpy as np
    import oracle
    t0 = time.perf_counter()
    idx, w, _, st = oracle.route_topk(logits, bias, wl.k, wl.n_group, wl.topk_group,
                                      wl.group_score, wl.bias_select_only)
    keep, _ = oracle.capacity_clip(idx, w, wl.E, wl.capacity)
    tc = wl.T // wl.n_chunks
    lays = [oracle.dispatch_layout(idx, keep, wl.E, wl.ep, c * tc, tc) for c in range(wl.n_chunks)]
    if is_mx(wl):
        xq, xs = oracle.quantize_blocks(x_np, 32)
        xrs = [oracle.permute(xq, lay["recv_token"]) for lay in lays]
    elif wl.ffn_fp8:
        xq, xs = oracle.quantize_rows(x_np)
        xrs = [oracle.permute(xq, lay["recv_token"]) for lay in lays]
    else:
        xrs = [oracle.permute(x_np, lay["recv_token"]) for lay in lays]
    t_index = time.perf_counter() - t0
    # rows of the sampled tokens (they sit in chunk 0)
    lay = lays[0]
    rows = [(p, e) for e in range(wl.E) for p in range(int(lay["expert_offsets"][e]), int(lay["expert_offsets"][e + 1]))
            if lay["recv_token"][p] < sample_tokens]
    weights = {e: fetch_expert(e) for e in sorted({e for _, e in rows})}   # host copies, untimed
    N = lay["N"]
    y = np.zeros((max(N, 1), wl.H), x_np.dtype)
    ye = np.zeros((max(N, 1), wl.H), np.float64)
    def row(p, e):
        if is_mx(wl):
            _, _, _, y[p], ye[p] = oracle.ffn_row_fp8_blocked(xrs[0][p], xs[lay["recv_token"][p]], *weights[e], 32)
        elif wl.ffn_fp8:
            _, _, _, y[p], ye[p] = oracle.ffn_row_fp8(xrs[0][p], xs[lay["recv_token"][p]], *weights[e])
        else:
            _, y[p], ye[p] = oracle.ffn_row(xrs[0][p], weights[e][0], weights[e][1])
    by_expert = {}
    for p, e in rows:
        by_expert.setdefault(e, []).append(p)
    t1 = time.perf_counter()
    oracle_rows(row, by_expert, threads)
    sub_pos = lay["pos"][:sample_tokens]
    ys = None
    if shared is not None:
        _, ys, _ = oracle.shared_expert(x_np[:sample_tokens], shared[0], shared[1])
    if wl.reduce_dense:
        oracle.combine_exact(ye, sub_pos, w, wl.T, x_np.dtype, y_shared=ys)
    else:
        oracle.combine(y, sub_pos, w, wl.T, y_shared=ys)
    t_ffn = time.perf_counter() - t1
    layer_s = t_index + t_ffn * (wl.T / sample_tokens)
    desc = (f"oracle route+clip+layout+permute over all {wl.T} tokens ({t_index:.2f} s, one thread), "
            f"FFN+combine for the {len(rows)} rows of the first {sample_tokens} tokens ({t_ffn:.2f} s, "
            f"rows in {threads} threads), extrapolated linearly to {wl.T} tokens")
    return wl.T / layer_s, t_index + t_ffn, desc


def fp8_expert(w13_e, w2_e, blocks=False):
    """The oracle's codes and scales of one expert's bf16 weights (host uint16
    bits): (w13 codes, w13 scales, w2 codes, w2 scales); one scale per row, or
    with blocks one per row and 32 values."""
    import oracle
    q = (lambda a: oracle.quantize_blocks(a, 32)) if blocks else oracle.quantize_rows
    a, sa = q(w13_e)
    b, sb = q(w2_e)
    return a, sa, b, sb


def oracle_row_seconds(wl):
    """Measured oracle cost of one FFN row, scaled from H = 2048, I = 768: bf16
    7.7 ms, FP8 with row scales 3 ms, FP8 with block scales 4.6 ms."""
    base = 4.6e-3 if is_mx(wl) else 3.0e-3 if wl.ffn_fp8 else 7.7e-3
    return base * (wl.H * wl.I) / (2048 * 768)


def sample_tokens_for(wl, seconds):
    # measured oracle cost of one FFN row at H = 2048, I = 768 (bf16 / FP8)
    row_s = oracle_row_seconds(wl)
    s = int(seconds / (wl.k * row_s))
    return max(1, min(wl.T // wl.n_chunks, s))


# --------------------------------------------------------------------------- arms

def reference_tokens(wl, seconds):
    """Tokens of one reference step: about `seconds` of oracle FFN rows, a
    multiple of the logical EP size (each source rank gets an equal block)."""
    row_s = oracle_row_seconds(wl)
    n = int(seconds / (wl.k * row_s)) // wl.ep * wl.ep
    return max(wl.ep, min(wl.T, n))


def reference_step(wl, Ts, logits, bias, x_np, fetch, threads=1):
    """The oracle's whole layer over the first Ts tokens of the workload, one chunk
    (a capacity scales with the sub-batch: ceil(C * Ts / T)), the FFN rows spread
    over `threads` host threads.  Expert weights are fetched (untimed) between the
    index steps and the FFN.  Returns seconds."""
    import numpy as np
    import oracle
    cap = wl.capacity if wl.capacity < 0 else -(-wl.capacity * Ts // wl.T)
    t0 = time.perf_counter()
    idx, w, _, st = oracle.route_topk(logits[:Ts], None if bias is None else bias, wl.k, wl.n_group,
                                      wl.topk_group, wl.group_score, wl.bias_select_only)
    keep, _ = oracle.capacity_clip(idx, w, wl.E, cap)
    lay = oracle.dispatch_layout(idx, keep, wl.E, wl.ep, 0, Ts)
    if is_mx(wl):
        xq, xs = oracle.quantize_blocks(x_np[:Ts], 32)
        xr = oracle.permute(xq, lay["recv_token"])
    elif wl.ffn_fp8:
        xq, xs = oracle.quantize_rows(x_np[:Ts])
        xr = oracle.permute(xq, lay["recv_token"])
    else:
        xr = oracle.permute(x_np[:Ts], lay["recv_token"])
    t_index = time.perf_counter() - t0
    eoff = lay["expert_offsets"]
    weights = {e: fetch(e) for e in range(wl.E) if eoff[e + 1] > eoff[e]}
    N = lay["N"]
    y = np.zeros((max(N, 1), wl.H), x_np.dtype)
    ye = np.zeros((max(N, 1), wl.H), np.float64)
    def row(p, e):
        wt = weights[e]
        if is_mx(wl):
            _, _, _, y[p], ye[p] = oracle.ffn_row_fp8_blocked(xr[p], xs[lay["recv_token"][p]], *wt, 32)
        elif wl.ffn_fp8:
            _, _, _, y[p], ye[p] = oracle.ffn_row_fp8(xr[p], xs[lay["recv_token"][p]], *wt)
        else:
            _, y[p], ye[p] = oracle.ffn_row(xr[p], wt[0], wt[1])
    t1 = time.perf_counter()
    oracle_rows(row, {e: range(int(eoff[e]), int(eoff[e + 1])) for e in weights}, threads)
    if wl.reduce_dense:
        oracle.combine_exact(ye, lay["pos"], w, Ts, x_np.dtype)
    else:
        oracle.combine(y, lay["pos"], w, Ts)
    return t_index + (time.perf_counter() - t1)


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import numpy as np
    import torch
    from combine_moe_route_12_b200.workload import make_inputs
    wl = workload_of(args)
    # inputs drawn on the CPU generator (no GPU needed for this arm); the expert
    # weights come from their own CPU generator, drawn expert by expert on first
    # use (same distribution as the GPU arm's, not the same values)
    torch.manual_seed(0)
    inp = make_inputs(wl, "cpu", seed=args.seed, weights=False)
    g = torch.Generator().manual_seed(wl.seed + 1)
    std = 1.0 / math.sqrt(wl.H)
    cache = {}
    conv = (lambda t: t.view(torch.int16).numpy().view(np.uint16).copy()) if wl.dtype == "bf16" \
        else (lambda t: t.numpy().copy())

    def fetch(e):
        if e not in cache:
            a = (torch.randn(2 * wl.I, wl.H, generator=g) * std).to(wl.torch_dtype)
            b = (torch.randn(wl.H, wl.I, generator=g) * std).to(wl.torch_dtype)
            cache[e] = fp8_expert(conv(a), conv(b), is_mx(wl)) if wl.ffn_fp8 else (conv(a), conv(b))
        return cache[e]

    logits = inp.logits.numpy()
    bias = None if inp.bias is None else inp.bias.numpy()
    x_np = conv(inp.x)
    threads = host_threads()
    Ts = reference_tokens(wl, 2.0 * threads)
    secs = []
    for i in range(args.warmup + args.steps):
        t = reference_step(wl, Ts, logits, bias, x_np, fetch, threads)
        if i >= args.warmup:
            secs.append(t)
    step_s = statistics.mean(secs)
    value = Ts / step_s
    desc = (f"each step: the oracle's whole layer (route, clip, layout, permute, FFN, combine) over the "
            f"first {Ts} of the {wl.T} tokens in one chunk, the FFN rows in {threads} threads, "
            f"{step_s:.2f} s (timed without the untimed draw of the routed experts' weights)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * step_s,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(wl, n, graph=None):
    return {"workload": wl.name, "T": wl.T, "H": wl.H, "E": wl.E, "k": wl.k, "I": wl.I,
            "ep_logical": wl.ep, "capacity": wl.capacity, "dispatch_chunks": wl.n_chunks,
            "decode_reduce": wl.reduce_dense, "ffn_fp8": wl.ffn_fp8, "global_batch_tokens": wl.T * n,
            "parallelism": "replicas" if n > 1 else "single",
            "l2": f"flushed between timed steps ({L2_FLUSH_BYTES >> 20} MiB write)",
            "timed": ("CPU oracle" if graph is None else
                      "moe_forward_chunked" + (" replayed from a CUDA graph" if graph else " eager"))}


def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist
    rank, world, local_rank = dist_env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=180), device_id=dev)
    from combine_moe_route_12_b200 import moe
    from combine_moe_route_12_b200.workload import WORKLOADS, make_inputs
    wl = workload_of(args)
    cfg = moe.config_from_workload(wl)
    peaks, peak_src = load_peaks()
    inp = make_inputs(wl, dev, seed=args.seed)
    torch.cuda.synchronize()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    sampler = ClockSampler(local_rank)
    sampler.start()

    # ---------------- timed region: K layer passes
    # The layer entry point (moe_forward_chunked: both streams, all chunks), by
    # default captured once into a CUDA graph and replayed, so that the host
    # launch cost of the small index kernels stays out of the GPU timeline.
    B = StepBuffers(moe, wl, cfg, dev)
    layer = moe.MoELayer(cfg, dev, host_splits=False)
    out_fw = torch.empty(wl.T, wl.H, dtype=wl.torch_dtype, device=dev)
    use_graph = not args.no_graph
    # FP8 FFN: the weights are quantised once, before any timing
    fp8 = None
    w13_l, w2_l, w13_sc, w2_sc = inp.w13, inp.w2, None, None
    if wl.ffn_fp8:
        q = moe.quantize_fp8_blocks if is_mx(wl) else moe.quantize_fp8
        w13_l, w13_sc = q(inp.w13)
        w2_l, w2_sc = q(inp.w2)
        fp8 = (w13_l, w13_sc, w2_l, w2_sc)
        torch.cuda.synchronize()

    def layer_pass():
        layer.forward(inp.logits, inp.bias, inp.x, w13_l, w2_l, out_fw,
                      w13_shared=inp.w13s, w2_shared=inp.w2s, w13_scale=w13_sc, w2_scale=w2_sc)

    for _ in range(max(args.warmup, 1)):
        flush.fill_(1)
        layer_pass()
    torch.cuda.synchronize()
    graph = None
    if use_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            layer_pass()
        torch.cuda.synchronize()
        for _ in range(args.warmup):
            flush.fill_(1)
            graph.replay()
        torch.cuda.synchronize()
    run = graph.replay if graph is not None else layer_pass
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for i in range(args.steps):
        flush.fill_(1)
        evs[i][0].record()
        run()
        evs[i][1].record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    total_ms = max_over_ranks(sum(step_ms), dev)
    if moe.moe_device_status(layer.ws) != 0:
        raise RuntimeError("device status bits set during the timed region")

    # ---------------- the two-stream overlap: the same layer with both of its
    # streams the same one (every kernel serialised), replayed from its own graph
    overlap = None
    if wl.n_chunks > 1 and not args.no_overlap:
        def one_stream_pass():
            # the stream current at the call (inside a capture: the capturing one)
            s_one = torch.cuda.current_stream()
            moe.moe_forward_chunked(cfg, inp.logits, inp.bias, inp.x, w13_l, w2_l, out_fw,
                                    layer.topk_idx, layer.topk_w, layer.keep, None, layer.ws,
                                    s_one, s_one, inp.w13s, inp.w2s, w13_sc, w2_sc)

        one_stream_pass()
        torch.cuda.synchronize()
        g1 = None
        if use_graph:
            g1 = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g1):
                one_stream_pass()
            torch.cuda.synchronize()
        run1 = g1.replay if g1 is not None else one_stream_pass
        for _ in range(args.warmup):
            flush.fill_(1)
            run1()
        # the two forms alternate, step by step, so that both see the same clocks
        # (the long steps run under the power cap)
        ev1 = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
        for i in range(args.steps):
            flush.fill_(1)
            ev1[i][0].record()
            run1()
            ev1[i][1].record()
            flush.fill_(1)
            ev1[i][2].record()
            run()
            ev1[i][3].record()
        torch.cuda.synchronize()
        if moe.moe_device_status(layer.ws) != 0:
            raise RuntimeError("device status bits set during the one-stream pass")
        one_ms = sum(e[0].elapsed_time(e[1]) for e in ev1) / args.steps
        two_ms = sum(e[2].elapsed_time(e[3]) for e in ev1) / args.steps
        del g1
        overlap = {"one_stream_ms": round(one_ms, 4), "two_stream_ms": round(two_ms, 4),
                   "timing": "one-stream and two-stream replays alternated step by step"}

    # ---------------- per-stage breakdown: the same kernels through the step ABI
    stage_ms, disp_ms, eager_step_ms, breakdown_mode = breakdown(
        moe, wl, cfg, inp, B, fp8, args.steps, flush, use_graph)
    idx_ms = index_path_ms(moe, wl, cfg, inp, B, args.steps, flush) if use_graph else None
    n_kept, n_active, tokens_read = layout_counts(moe, wl, cfg, B)
    alg = algorithmic(wl, n_kept, n_active, tokens_read)
    bwd = backward_row_passes(moe, wl, cfg, B, n_kept[-1], peaks, flush, args) \
        if args.backward and not wl.reduce_dense else None
    lbwd = layer_backward(moe, wl, cfg, inp, layer, flush, args, peaks, peak_src) \
        if args.backward and not wl.reduce_dense and not wl.ffn_fp8 else None
    if overlap is not None:
        # what the second stream can hide: the dispatch (layout + permute) of
        # every chunk after the first, which runs beside the previous chunk's FFN
        hideable = sum(disp_ms[1:])
        hidden = overlap["one_stream_ms"] - overlap["two_stream_ms"]
        overlap.update({"dispatch_ms_per_chunk": [round(v, 4) for v in disp_ms],
                        "hideable_ms": round(hideable, 4), "hidden_ms": round(hidden, 4),
                        "hidden_frac": hidden / hideable if hideable > 0 else None,
                        "note": "one_stream: moe_forward_chunked with s_dispatch = s_compute (same "
                                "kernels, serialised); hideable: dispatch_layout + permute of chunks "
                                ">= 1 from the breakdown"})

    # ---------------- the same layer in one chunk: the FFN reads each expert's
    # weights once per layer pass (the tensor-roof reading of a chunked workload)
    unchunked = None
    if wl.n_chunks > 1 and not args.no_unchunked:
        wl1 = wl.with_(n_chunks=1)
        cfg1 = moe.config_from_workload(wl1)
        B1 = StepBuffers(moe, wl1, cfg1, dev)
        st1, _, step1, _ = breakdown(moe, wl1, cfg1, inp, B1, fp8, args.steps, flush, use_graph)
        k1, a1, r1 = layout_counts(moe, wl1, cfg1, B1)
        alg1 = algorithmic(wl1, k1, a1, r1)
        unchunked = {"roofline": ffn_roofline(wl1, alg1, st1["grouped_ffn"], peaks, peak_src, None),
                     "dispatch_combine": dispatch_combine(alg1, st1, peaks, peak_src),
                     "stage_ms": {k: round(v, 4) for k, v in st1.items()},
                     "breakdown_step_ms": round(step1, 4)}
        del B1
        torch.cuda.empty_cache()

    # ---------------- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        h_logits = inp.logits.cpu().pin_memory()
        h_x = inp.x.cpu().pin_memory()
        h_bias = None if inp.bias is None else inp.bias.cpu().pin_memory()
        h_out = torch.empty(wl.T, wl.H, dtype=wl.torch_dtype).pin_memory()
        # moe_forward_host: the copies in and out are the library's, inside the call
        layer_h = moe.MoELayer(cfg, dev, host_splits=False, host_io=True)
        e2e_ms = 0.0
        for i in range(args.warmup + args.steps):
            flush.fill_(1)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            layer_h.forward_host(h_logits, h_bias, h_x, w13_l, w2_l, h_out,
                                 w13_shared=inp.w13s, w2_shared=inp.w2s, w13_scale=w13_sc,
                                 w2_scale=w2_sc)
            b.record()
            b.synchronize()
            if i >= args.warmup:
                e2e_ms += a.elapsed_time(b)
        if moe.moe_device_status(layer_h.ws) != 0:
            raise RuntimeError("device status bits set during the host-buffer pass")
        if not torch.equal(h_out, out_fw.cpu()):
            raise RuntimeError("the host-buffer forward differs from the device forward")
        e2e_ms = max_over_ranks(e2e_ms, dev)
        h2d = h_logits.numel() * 4 + h_x.numel() * h_x.element_size() + (0 if h_bias is None else h_bias.numel() * 4)
        d2h = h_out.numel() * h_out.element_size()
        e2e = {"value": world * wl.T * args.steps / (e2e_ms / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}
    sampler.stop()
    clocks = sampler.summary()

    # ---------------- CPU oracle on a bounded sample (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        conv = (lambda t: t.detach().cpu().view(torch.int16).numpy().view(np.uint16).copy()) \
            if wl.dtype == "bf16" else (lambda t: t.detach().cpu().numpy().copy())
        fetch = (lambda e: fp8_expert(conv(inp.w13[e]), conv(inp.w2[e]), is_mx(wl))) if wl.ffn_fp8 else \
            (lambda e: (conv(inp.w13[e]), conv(inp.w2[e])))
        threads = host_threads()
        s_tok = sample_tokens_for(wl, 15.0 * threads)
        shared = None if inp.w13s is None else (conv(inp.w13s), conv(inp.w2s))
        v, secs, desc = oracle_sample(wl, inp.logits.cpu().numpy(),
                                      None if inp.bias is None else inp.bias.cpu().numpy(),
                                      conv(inp.x), fetch, s_tok, shared, threads)
        cpu = {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc,
               "cpu_seconds": round(secs, 2)}

    if rank == 0:
        ms_per_step = total_ms / args.steps
        value = world * wl.T * args.steps / (total_ms / 1e3)
        src = kernel_src_hash(wl.ffn_fp8, is_mx(wl))
        tr = FFN_TRAFFIC.get(wl.name)
        traffic = tr["bytes"] if tr and tr.get("src") == src and tr.get("chunks", 1) == wl.n_chunks else None
        roof = ffn_roofline(wl, alg, stage_ms["grouped_ffn"], peaks, peak_src, traffic)
        dc = dispatch_combine(alg, stage_ms, peaks, peak_src)
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "e4m3 (expert FFN) / bf16" if wl.ffn_fp8 else wl.dtype, "data": "synthetic",
            "config": workload_config(wl, world, use_graph),
            "roofline": roof,
            "dispatch_combine": dc,
            "ffn_tflops": roof["tflops"],
            "ffn_gbs": roof["gbs"],
            "stage_ms": {k: round(v, 4) for k, v in stage_ms.items()},
            "breakdown_step_ms": round(eager_step_ms, 4),
            "breakdown_mode": breakdown_mode,
            "index_path": None if idx_ms is None else {
                "ms": round(idx_ms, 4),
                "what": "route + clip + the first chunk's dispatch layout as one CUDA graph (no events "
                        "inside), L2 flushed before each replay"},
            "kept_rows": alg["N"],
            "e2e": e2e,
            "cpu_baseline": cpu,
            "gpu_launches": kernels_per_step(wl) * args.steps,
            "clocks": clocks,
        }
        if unchunked is not None:
            line["roofline_unchunked"] = unchunked
        if overlap is not None:
            line["overlap"] = overlap
        if bwd is not None:
            line["backward_row_passes"] = bwd
        if lbwd is not None:
            line["backward"] = lbwd
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
