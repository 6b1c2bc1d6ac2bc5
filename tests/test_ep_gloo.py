"""Host side of the expert-parallel exchange (`combine_moe_route_12_b200.ep`) on
CPU: world-size-2 and -3 gloo process groups stand in for the NCCL ranks (the
same torch.distributed calls).  Checked: the split counts taken from a layout's
expert offsets, the count-table all-to-all (row d to rank d), the variable
all-to-all of rows (each source's rows for this rank, source after source, in
the order sent, empty segments included), and that the reverse exchange returns
every row to its sender in its original place."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from combine_moe_route_12_b200 import ep


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_split_counts_from_expert_offsets():
    # 8 experts over 2 ranks; expert 5 empty
    counts = [3, 0, 2, 1, 4, 0, 2, 5]
    eoff = [0]
    for c in counts:
        eoff.append(eoff[-1] + c)
    sizes, table = ep.split_counts(eoff, 2)
    assert sizes == [6, 11]
    assert table == [[3, 0, 2, 1], [4, 0, 2, 5]]
    sizes, table = ep.split_counts(eoff, 4)
    assert sizes == [3, 3, 4, 7] and table == [[3, 0], [2, 1], [4, 0], [2, 5]]
    assert ep.split_counts([0, 0, 0], 1) == ([0], [[0, 0]])


def _table(src, world, El):
    """Rows that rank `src` sends each destination, per local expert (seeded; some zero)."""
    g = torch.Generator().manual_seed(1000 + src)
    t = torch.randint(0, 4, (world, El), generator=g, dtype=torch.int32)
    t[(src + 1) % world, 0] = 0
    return t


def _rows(src, table, H):
    """The send buffer of `src`: row values name (source, destination, expert, index)."""
    out = []
    world, El = table.shape
    for d in range(world):
        for e in range(El):
            for i in range(int(table[d, e])):
                out.append([src, d, e, i] + [src * 1000 + d * 100 + e * 10 + i] * (H - 4))
    return torch.tensor(out, dtype=torch.float32).reshape(-1, H)


def _worker(rank, world, port, q):
    import torch.distributed as dist
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        El, H = 3, 8
        send_counts = _table(rank, world, El)
        recv_counts = ep.exchange_counts(send_counts)
        for s in range(world):
            assert torch.equal(recv_counts[s], _table(s, world, El)[rank]), "count table row from source s"
        rows = _rows(rank, send_counts, H)
        send_sizes = send_counts.sum(1).tolist()
        recv_sizes = [sum(r) for r in recv_counts.tolist()]
        got = ep.exchange_rows(rows, send_sizes, recv_sizes)
        want = []
        for s in range(world):
            t = _table(s, world, El)
            for e in range(El):
                for i in range(int(t[rank, e])):
                    want.append([s, rank, e, i])
        assert got.shape == (sum(recv_sizes), H)
        assert got[:, :4].tolist() == [[float(v) for v in w] for w in want]
        # the reverse exchange brings every row back to its place
        back = ep.exchange_rows(got, recv_sizes, send_sizes)
        assert torch.equal(back, rows)
        q.put((rank, "ok"))
        dist.barrier()
    except AssertionError as exc:
        q.put((rank, f"fail: {exc}"))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_exchange_counts_and_rows_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == [(r, "ok") for r in range(world)]
