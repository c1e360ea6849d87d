"""The multi-rank plumbing of bench.py on CPU: two gloo ranks.

With N > 1 GPUs the bench runs one independent layer per rank (no data-path
collective).  What the ranks share is host logic: the rendezvous, the barrier
around the timed region, the max over ranks of the device time, and the rule
that only rank 0 runs and prints the reference arm.  Those run here on two
gloo processes, with no GPU.
"""

import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist

    class A:
        impl = "reference"
    r, w, _ = bench.setup_dist(A())
    try:
        assert (r, w) == (rank, world) and dist.get_backend() == "gloo"
        bench.barrier(w)
        m = bench.max_over_ranks(10.0 + 5.0 * rank, w)          # per-rank step times
        ref = bench.run_reference(A(), r, w) if r != 0 else "rank0"
        out.put((rank, m, ref))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_only_rank0_reports():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [m for _, m, _ in res] == [15.0, 15.0]
    assert res[1][2] is None            # rank 1 does no reference work and prints nothing
