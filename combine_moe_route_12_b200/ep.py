"""Expert parallelism over real ranks: one process per GPU, the EP group a
torch.distributed process group (NCCL on GPUs).

The exchange the pages describe (axolotl docs, integrations.expert_parallel.args:
`expert_parallel_backend = torch`, `all_to_all_single` over the EP group, with the
host-side split counts kept): experts are owned by contiguous blocks of E / ep per
rank, each rank routes its own tokens, and

  dispatch   route + clip + dispatch layout (destination ranks = the EP group) +
             permute, locally: the send buffer holds, destination after
             destination, the rows of that destination's experts in (expert, token)
             order;
  counts     all-to-all of the per-(destination, local expert) row counts; the
             host copies give the variable all-to-all its split sizes;
  rows       all-to-all of the rows;
  experts    regroup the received rows expert after expert (moe_ep_regroup), the
             grouped SwiGLU FFN over the local experts, regroup back;
  rows back  the reverse all-to-all of the expert outputs;
  combine    the weighted combine of each token's rows, locally.

Every arithmetic step is one of the library's kernels; this module holds the
buffers and the collective calls.  The phases are separate methods so that a
test can run several ranks' phases in one process and move the rows between them
itself.  Scope: the routed experts without a capacity and without the decode
form's dense reduce (the capacity is a per-forward limit over every rank's
tokens, which needs a global exchange of counts before the clip; the decode
reduce writes into the token's home rank).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import moe


@dataclass
class DispatchState:
    """What the dispatch phase leaves for the exchange and the combine."""
    topk_w: torch.Tensor
    pos: torch.Tensor
    xr: torch.Tensor             # [N, H] send buffer, destination after destination
    n_rows: int                  # N
    send_counts: torch.Tensor    # device int32 [ep, E // ep]: rows per (destination, its local expert)
    send_sizes: list             # host: rows per destination (the split sizes)


class EPRank:
    """One rank of an EP group of `ep` ranks: its own T tokens, experts
    [rank * E / ep, (rank + 1) * E / ep) with weights w13 [E / ep, 2I, H] and
    w2 [E / ep, H, I] in the layer dtype."""

    def __init__(self, T: int, H: int, E: int, k: int, I: int, ep: int, rank: int, dtype="bf16",
                 device="cuda"):
        if E % ep:
            raise ValueError("E must be a multiple of the EP group size")
        self.T, self.H, self.E, self.k, self.I, self.ep, self.rank = T, H, E, k, I, ep, rank
        self.El = E // ep
        self.dev = torch.device(device)
        # routing and layout over the whole group's experts, destinations = the group
        self.cfg = moe.make_config(T, H, E, k, I, ep, -1, dtype)
        moe.config_check(self.cfg)
        self.dtype = torch.float32 if dtype in ("f32", moe.MOE_F32) else torch.bfloat16
        self.ws = moe.alloc_workspace(moe.workspace_bytes(self.cfg), self.dev)
        # the grouped FFN over this rank's experts: the rows it can receive are at
        # most every rank's tokens times k
        self.cfg_local = moe.make_config(max(1, T * ep), H, self.El, k, I, 1, -1, dtype)
        moe.config_check(self.cfg_local)
        self.ws_local = moe.alloc_workspace(moe.workspace_bytes(self.cfg_local), self.dev)
        d = self.dev
        self.topk_idx = torch.empty(T, k, dtype=torch.int32, device=d)
        self.topk_w = torch.empty(T, k, dtype=torch.float32, device=d)
        self.counts = torch.empty(E, dtype=torch.int32, device=d)
        self.keep = torch.empty(T, k, dtype=torch.uint8, device=d)
        self.kept = torch.empty(E, dtype=torch.int32, device=d)
        self.eoff = torch.empty(E + 1, dtype=torch.int32, device=d)
        self.roff = torch.empty(ep + 1, dtype=torch.int32, device=d)
        nmax = max(1, moe.max_recv_rows(self.cfg, T))
        self.recv_token = torch.empty(nmax, dtype=torch.int32, device=d)
        self.recv_slot = torch.empty(nmax, dtype=torch.int32, device=d)
        self.pos = torch.empty(T, k, dtype=torch.int32, device=d)
        self.splits = torch.empty(ep, ep, dtype=torch.int32, device=d)
        self.splits_host = torch.zeros(E + 1 + ep * ep, dtype=torch.int32, pin_memory=True)
        self.xr = torch.empty(nmax, H, dtype=self.dtype, device=d)
        self.local_offsets = torch.empty(self.El + 1, dtype=torch.int32, device=d)

    # ------------------------------------------------------------------ phases

    def dispatch(self, logits, bias, x) -> DispatchState:
        """Route, clip (no capacity: every slot kept), lay out by destination rank
        and permute this rank's tokens.  Synchronises on the layout's host copy of
        the expert offsets (the split sizes)."""
        c = self.cfg
        moe.moe_route_topk(c, logits, bias, self.topk_idx, self.topk_w, self.counts, self.ws)
        moe.moe_capacity_clip(c, self.topk_idx, self.topk_w, self.counts, self.keep, self.kept, self.ws)
        moe.moe_dispatch_layout(c, 0, self.T, self.topk_idx, self.keep, self.eoff, self.roff, self.recv_token,
                                self.recv_slot, self.pos, self.splits, self.splits_host, self.ws)
        moe.moe_permute(c, x, self.pos, 0, self.T, self.xr)
        torch.cuda.current_stream(self.dev).synchronize()
        eoff = self.splits_host[:self.E + 1].tolist()
        send_sizes, table = split_counts(eoff, self.ep)
        send_counts = torch.tensor(table, dtype=torch.int32).to(self.dev)
        return DispatchState(self.topk_w, self.pos, self.xr, eoff[self.E], send_counts, send_sizes)

    def experts(self, rows_recv, recv_counts, w13, w2):
        """The expert phase on the rows received from every source (source-major,
        recv_counts device int32 [ep, E / ep]): regroup expert-major, the grouped
        SwiGLU FFN over the local experts, regroup back.  Returns the outputs in the
        received order."""
        n = rows_recv.shape[0]
        xl = torch.empty(max(n, 1), self.H, dtype=self.dtype, device=self.dev)
        moe.moe_ep_regroup(self.cfg, recv_counts, rows_recv, xl, n, 0, self.ws, self.local_offsets)
        h = torch.empty(max(n, 1), self.I, dtype=self.dtype, device=self.dev)
        yl = torch.empty(max(n, 1), self.H, dtype=self.dtype, device=self.dev)
        moe.moe_grouped_swiglu_ffn(self.cfg_local, n, xl, self.local_offsets, w13, w2, h, yl, None, None, None,
                                   None, self.ws_local)
        y = torch.empty(max(n, 1), self.H, dtype=self.dtype, device=self.dev)
        moe.moe_ep_regroup(self.cfg, recv_counts, yl, y, n, 1, self.ws)
        return y[:n]

    def combine(self, st: DispatchState, y_back, out):
        """Each token's weighted sum of its rows' outputs (returned in the send
        buffer's order)."""
        moe.moe_combine(self.cfg, y_back, st.pos, st.topk_w, 0, self.T, out)
        return out

    def status(self) -> int:
        """The device status bits of both workspaces (cleared)."""
        return moe.moe_device_status(self.ws) | moe.moe_device_status(self.ws_local)

    # ------------------------------------------------------------------ whole layer

    def forward(self, logits, bias, x, w13, w2, out, group=None):
        """The layer on this rank's tokens; every rank of `group` (the EP group, of
        size ep, this rank at index rank) calls it with its own tokens and experts."""
        st = self.dispatch(logits, bias, x)
        recv_counts = exchange_counts(st.send_counts, group)
        recv_sizes = [sum(r) for r in recv_counts.cpu().tolist()]   # host split sizes
        rows_recv = exchange_rows(st.xr[:st.n_rows], st.send_sizes, recv_sizes, group)
        y = self.experts(rows_recv, recv_counts, w13, w2)
        y_back = exchange_rows(y, recv_sizes, st.send_sizes, group)
        return self.combine(st, y_back, out)


# ---------------------------------------------------------------------- exchanges

def split_counts(expert_offsets, ep: int):
    """The host-side split counts of one rank's send buffer, from the dispatch
    layout's expert offsets (E + 1 values, experts owned by contiguous blocks of
    E / ep per rank): (rows for each destination, [ep][E / ep] rows for each
    destination's local experts)."""
    E = len(expert_offsets) - 1
    El = E // ep
    sizes = [expert_offsets[(d + 1) * El] - expert_offsets[d * El] for d in range(ep)]
    table = [[expert_offsets[d * El + e + 1] - expert_offsets[d * El + e] for e in range(El)]
             for d in range(ep)]
    return sizes, table


def exchange_counts(send_counts: torch.Tensor, group=None) -> torch.Tensor:
    """All-to-all of the [ep, E / ep] count table: row d goes to rank d; returns
    the table of what every source sends this rank (row s from source s)."""
    import torch.distributed as dist
    recv = torch.empty_like(send_counts)
    dist.all_to_all_single(recv, send_counts.contiguous(), group=group)
    return recv


def exchange_rows(rows: torch.Tensor, send_sizes, recv_sizes, group=None) -> torch.Tensor:
    """Variable all-to-all of rows: send_sizes[d] rows to rank d, in order;
    returns recv_sizes[s] rows from each source s, source after source."""
    import torch.distributed as dist
    out = torch.empty(sum(recv_sizes), *rows.shape[1:], dtype=rows.dtype, device=rows.device)
    dist.all_to_all_single(out, rows.contiguous(), output_split_sizes=list(recv_sizes),
                           input_split_sizes=list(send_sizes), group=group)
    return out
