"""Seeded synthetic workloads for the expert-parallel MoE layer hot path.

This module only *describes* workloads and draws their random inputs.  It holds
none of the layer's arithmetic (no routing, no clipping, no layout, no FFN, no
combine), so both the CUDA path and the CPU oracle can be fed from it.

The five workloads restate the layer shapes that the expert-parallel pages
discuss:

* ``tiny``            - T=256, H=128, E=8, k=2, I=256, fp32, 2 logical EP ranks,
                        no capacity.  Small enough for the oracle to run whole.
* ``qwen3_30b_a3b``   - Qwen3-30B-A3B-shaped layer: T=4096 (one 4k packed
                        sequence), H=2048, E=128, k=8, I=768, bf16, EP=2.
* ``skew_capacity``   - same shapes at T=16384 with a skewed router (per-expert
                        bias 3*ln p_r, p_r a Zipf(1.2) mass over a random
                        permutation of experts) and a per-expert capacity of
                        1024 assignments (axolotl ExpertParallelArgs,
                        ``expert_parallel_token_capacity``), EP=4.
* ``dsv3_prefill``    - DeepSeek-V3-shaped prefill: T=8192, H=7168, E=256, k=8,
                        I=2048, bf16, EP=8, two dispatch chunks (axolotl
                        ``expert_parallel_dispatch_chunks``).
* ``dsv3_decode``     - DeepSeek-V3-shaped decode step: T=256, same shapes,
                        EP=64, capacity 1024 (never binding), expert outputs
                        reduced straight into a dense [T, H] output (LightLLM
                        PR 1687, decode reduce).

Input recipe (the pages fix none of it; every choice is a stated reading):

* x ~ N(0, 1); router weight W_r and every expert weight ~ N(0, 1/H)
  (W_down included, although its fan-in is I).
* bf16 workloads round x and the weights to bf16 (round to nearest even) after
  drawing them in fp32.
* router logits = x @ W_r in fp32 (x after its bf16 rounding), computed once
  here and handed identically to both implementations.  The router GEMM is not
  part of the hot path.
* the skewed workload adds bias[e] = 3 * ln(p_{rank(e)}), p_r proportional to
  r^-1.2 for r = 1..128 and normalised, with rank(e) a seeded permutation.
* a workload with ``shared_I`` > 0 also draws a shared expert, w13s [2 I_s, H]
  and w2s [H, I_s] ~ N(0, 1/H), from its own seeded generator.
* ``dsv3_grouped`` (routing variants, DSV3 prefill shape in one chunk): grouped
  top-k with 8 groups of 32 experts and 4 kept per token (group score: the sum
  of a group's two best biased logits), and a load-balancing-like bias
  bias[e] ~ N(0, 0.5^2) (seeded) that steers the selection only.
* ``qwen3_30b_a3b_fp8`` and ``dsv3_prefill_fp8``: the Qwen3 and DSV3 prefill
  shapes with the expert FFN in FP8 (LightLLM PR 1687: FP8 grouped GEMM with
  UE8M0 scales); ``*_mxfp8``: the same with one scale per 32 K values.  Inputs are drawn exactly as for the bf16 workloads; the
  weights are quantised row by row to E4M3 codes with UE8M0 scales once, before
  the layer runs, and x per call inside it.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class MoEWorkload:
    name: str
    T: int
    H: int
    E: int
    k: int
    I: int
    dtype: str          # "f32" or "bf16": storage / arithmetic type of x, weights, h, y, out
    ep: int             # logical expert-parallel ranks
    capacity: int = -1  # < 0 means no cap
    n_chunks: int = 1
    reduce_dense: bool = False   # decode mode: y is reduced straight into out
    skew_bias: bool = False
    seed: int = 0
    # routing variants (grouped top-k, bias in the selection only)
    n_group: int = 0
    topk_group: int = 0
    group_score: int = 0          # 0: best logit of the group; 1: sum of its two best
    bias_select_only: bool = False
    balance_bias: bool = False    # a small per-expert bias ~ N(0, 0.5^2), the load-balancing kind
    shared_I: int = 0             # a shared expert of this intermediate size (0: none)
    ffn_fp8: int = 0              # the expert FFN on E4M3 codes: 1 with UE8M0 row scales,
                                  # 2 with one UE8M0 scale per 32 K values

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def with_(self, **kw) -> "MoEWorkload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny": MoEWorkload("tiny", T=256, H=128, E=8, k=2, I=256, dtype="f32", ep=2),
    "qwen3_30b_a3b": MoEWorkload("qwen3_30b_a3b", T=4096, H=2048, E=128, k=8, I=768,
                                 dtype="bf16", ep=2),
    "skew_capacity": MoEWorkload("skew_capacity", T=16384, H=2048, E=128, k=8, I=768,
                                 dtype="bf16", ep=4, capacity=1024, skew_bias=True),
    "dsv3_prefill": MoEWorkload("dsv3_prefill", T=8192, H=7168, E=256, k=8, I=2048,
                                dtype="bf16", ep=8, n_chunks=2),
    "dsv3_decode": MoEWorkload("dsv3_decode", T=256, H=7168, E=256, k=8, I=2048,
                               dtype="bf16", ep=64, capacity=1024, reduce_dense=True),
    # routing variants on the DSV3 prefill shape (one chunk): 8 groups of 32
    # experts, 4 kept per token by the sum of their two best biased logits, the
    # bias used for the selection only, and one shared expert of I = 2048
    "dsv3_grouped": MoEWorkload("dsv3_grouped", T=8192, H=7168, E=256, k=8, I=2048,
                                dtype="bf16", ep=8, n_group=8, topk_group=4, group_score=1,
                                bias_select_only=True, balance_bias=True, shared_I=2048),
    # the expert FFN in FP8 on the same shapes
    "qwen3_30b_a3b_fp8": MoEWorkload("qwen3_30b_a3b_fp8", T=4096, H=2048, E=128, k=8, I=768,
                                     dtype="bf16", ep=2, ffn_fp8=True),
    "dsv3_prefill_fp8": MoEWorkload("dsv3_prefill_fp8", T=8192, H=7168, E=256, k=8, I=2048,
                                    dtype="bf16", ep=8, n_chunks=2, ffn_fp8=True),
    # the expert FFN in FP8 with K-blocked scales (one per 32 values), h quantised
    # inside the SwiGLU epilogue
    "qwen3_30b_a3b_mxfp8": MoEWorkload("qwen3_30b_a3b_mxfp8", T=4096, H=2048, E=128, k=8, I=768,
                                       dtype="bf16", ep=2, ffn_fp8=2),
    "dsv3_prefill_mxfp8": MoEWorkload("dsv3_prefill_mxfp8", T=8192, H=7168, E=256, k=8, I=2048,
                                      dtype="bf16", ep=8, n_chunks=2, ffn_fp8=2),
}


@dataclass
class MoEInputs:
    """Inputs of one layer invocation.  ``w13`` is [E, 2I, H] (rows 0..I-1 gate,
    I..2I-1 up), ``w2`` is [E, H, I]; both row-major, K contiguous."""
    logits: torch.Tensor      # fp32 [T, E]
    bias: torch.Tensor | None  # fp32 [E] or None
    x: torch.Tensor           # [T, H]
    w13: torch.Tensor         # [E, 2I, H]
    w2: torch.Tensor          # [E, H, I]
    w13s: torch.Tensor | None = None   # shared expert [2 I_s, H]
    w2s: torch.Tensor | None = None    # shared expert [H, I_s]


def zipf_bias(E: int, s: float, gen: torch.Generator) -> torch.Tensor:
    """3*ln(p_rank(e)) with p_r proportional to r^-s over ranks 1..E and a seeded
    random rank permutation (skewed-router workload)."""
    r = torch.arange(1, E + 1, dtype=torch.float64)
    p = r.pow(-s)
    p = p / p.sum()
    perm = torch.randperm(E, generator=gen)
    bias = torch.empty(E, dtype=torch.float64)
    bias[perm] = 3.0 * torch.log(p)
    return bias.float()


def make_inputs(wl: MoEWorkload, device: str | torch.device = "cpu",
                seed: int | None = None, weights: bool = True) -> MoEInputs:
    """Draw one seeded set of inputs on ``device``.

    Values depend on the device's generator (CPU and CUDA streams differ); each
    test or benchmark draws once and feeds the same tensors to both sides.
    Weights are drawn one expert at a time so that the large workloads never
    hold an fp32 copy of all weights.
    """
    seed = wl.seed if seed is None else seed
    device = torch.device(device)
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    dt = wl.torch_dtype
    std = 1.0 / math.sqrt(wl.H)

    x32 = torch.randn(wl.T, wl.H, generator=g, device=device)
    x = x32.to(dt)
    wr = torch.randn(wl.H, wl.E, generator=g, device=device) * std
    logits = x.float() @ wr
    bias = None
    if wl.skew_bias:
        gb = torch.Generator(device="cpu")
        gb.manual_seed(seed + 7919)
        bias = zipf_bias(wl.E, 1.2, gb).to(device)
    elif wl.balance_bias:
        gb = torch.Generator(device="cpu")
        gb.manual_seed(seed + 104729)
        bias = (0.5 * torch.randn(wl.E, generator=gb)).to(device)

    if weights:
        w13 = torch.empty(wl.E, 2 * wl.I, wl.H, dtype=dt, device=device)
        w2 = torch.empty(wl.E, wl.H, wl.I, dtype=dt, device=device)
        for e in range(wl.E):
            w13[e] = (torch.randn(2 * wl.I, wl.H, generator=g, device=device) * std).to(dt)
            w2[e] = (torch.randn(wl.H, wl.I, generator=g, device=device) * std).to(dt)
    else:
        w13 = torch.empty(0, dtype=dt, device=device)
        w2 = torch.empty(0, dtype=dt, device=device)
    w13s = w2s = None
    if wl.shared_I > 0:
        # the shared expert draws from its own seeded stream, after the routed ones
        gs = torch.Generator(device=device)
        gs.manual_seed(seed + 15485863)
        w13s = (torch.randn(2 * wl.shared_I, wl.H, generator=gs, device=device) * std).to(dt)
        w2s = (torch.randn(wl.H, wl.shared_I, generator=gs, device=device) * std).to(dt)
    return MoEInputs(logits=logits.contiguous(), bias=bias, x=x.contiguous(),
                     w13=w13, w2=w2, w13s=w13s, w2s=w2s)
