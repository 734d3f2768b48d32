"""Expert parallelism, host side, on CPU: the send splits follow the expert offsets, and the
layer's two collectives (NcclExchange: torch.distributed all-to-all) move the count table
and rows with uneven splits correctly between 2 gloo ranks (127.0.0.1)."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_send_splits_follow_the_offsets():
    from top_routing_grouped_03_b200.ep import send_splits
    # 8 experts over 4 ranks (2 each); expert e received counts[e] rows
    counts = [3, 0, 5, 1, 0, 0, 7, 2]
    off = [0]
    for c in counts:
        off.append(off[-1] + c)
    assert send_splits(off, 4, 2) == [3, 6, 0, 9]
    assert send_splits(off, 1, 8) == [18]
    assert send_splits(off, 8, 1) == counts


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import sys
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from top_routing_grouped_03_b200.ep import NcclExchange
    ex = NcclExchange()
    El = 3
    # rank r sends count table row d = (10 r + d, ...) to rank d
    send_counts = torch.tensor([[10 * rank + d + e for e in range(El)] for d in range(world)],
                               dtype=torch.int32)
    recv_counts = ex.counts(send_counts)
    # rows: rank r sends r + d + 1 rows to rank d, each row = [r, d, i]
    send_splits = [rank + d + 1 for d in range(world)]
    rows = torch.tensor([[rank, d, i] for d in range(world) for i in range(rank + d + 1)],
                        dtype=torch.float32)
    recv_splits = [s + rank + 1 for s in range(world)]
    got = ex.rows(rows, send_splits, recv_splits)
    q.put((rank, recv_counts.tolist(), got.tolist()))
    dist.barrier()
    dist.destroy_process_group()


def test_exchange_moves_counts_and_uneven_rows_between_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 2
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict((r, (c, g)) for r, c, g in (q.get(timeout=120) for _ in procs))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        counts, got = res[r]
        # row s of what rank r received is source s's table row r
        assert counts == [[10 * s + r + e for e in range(3)] for s in range(world)]
        # rows arrive source by source, in the order each source sent them
        assert got == [[s, r, i] for s in range(world) for i in range(s + r + 1)]
