"""Host plumbing of bench.py's multi-GPU mode (replicas only), run as two
gloo ranks on the CPU: rendezvous, barrier, max-over-ranks timing and the
whole-job aggregate."""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, ws, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(ws),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    import bench
    n, r, local = bench.dist_init("gloo")
    assert (n, r, local) == (ws, rank, rank)
    bench.barrier(n)
    t = bench.reduce_max(1.0 + rank, n)            # rank 1 is the slower replica
    out[rank] = (t, bench.aggregate_gbps(n, 2e9, t))
    bench.barrier(n)
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_aggregate():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
        assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
        res = dict(out)
    # both ranks see the slowest rank's time; 2 replicas x 2 GB in 2 ms = 2000 GB/s
    assert res[0] == res[1] == (2.0, 2000.0)


def test_single_process_needs_no_process_group():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        os.environ.pop(k, None)
    assert bench.dist_init() == (1, 0, 0)
    assert bench.reduce_max(3.5, 1) == 3.5
    assert bench.aggregate_gbps(1, 1e9, 1.0) == 1000.0
