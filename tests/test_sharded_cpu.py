"""The exchanges of the head-sharded layer on CPU: gloo ranks moving
contiguous runs of rows between a sequence-sharded and a head-sharded layout.

Reference: the whole tensor, sliced.  Rank s holds rows [r0_s, r0_s + n_s) of
every head in its first n_s local rows (the rest is padding); after
seq_to_heads rank g holds every rank's rows of heads [g*hpr, (g+1)*hpr).
"""

import os
import socket
import sys

import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from dynamic_block_sparse_variance_b200.sharded import TorchDistExchange
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        heads, d, pad = 2 * world, 3, 2
        counts = [3 + 2 * s for s in range(world)]          # uneven row counts per rank (>= 2*world in total)
        starts = [sum(counts[:s]) for s in range(world)]
        total = sum(counts)
        g = torch.Generator().manual_seed(0)
        full = torch.randn(heads, total, d, generator=g)     # the same on every rank
        rows_of = lambda s: (starts[s], counts[s])
        ex = TorchDistExchange(rank, world)
        # records-style all-gather: equal shares, concatenated in rank order
        loc = full[0, 2 * rank:2 * rank + 2].contiguous()
        gathered = torch.empty(2 * world, d)
        ex.all_gather(loc, gathered)
        ok0 = torch.equal(gathered, full[0, :2 * world])
        # sequence -> heads
        x_loc = torch.full((heads, counts[rank] + pad, d), float("nan"))
        x_loc[:, :counts[rank]] = full[:, starts[rank]:starts[rank] + counts[rank]]
        hpr = heads // world
        x_h = torch.full((hpr, total, d), float("nan"))
        ex.seq_to_heads(x_loc, x_h, rows_of)
        ok1 = torch.equal(x_h, full[rank * hpr:(rank + 1) * hpr])
        # heads -> sequence, back into a fresh local buffer
        back = torch.full_like(x_loc, float("nan"))
        ex.heads_to_seq(x_h, back, rows_of)
        ok2 = torch.equal(back[:, :counts[rank]], x_loc[:, :counts[rank]])
        out.put((rank, ok0 and ok1, ok2))
    finally:
        dist.destroy_process_group()


def _run(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert all(ok1 and ok2 for _, ok1, ok2 in res), res


def test_exchanges_two_gloo_ranks():
    _run(2)


def test_exchanges_three_gloo_ranks():
    _run(3)
