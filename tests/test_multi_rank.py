"""bench.py's multi-rank plumbing on two host ranks (gloo): the rendezvous,
the barrier, the max- and sum-over-ranks reductions that the timing and the
whole-job value use, and the reference arm running on rank 0 only."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    r, w, _ = bench.dist_init()
    bench.barrier(w)
    mx = bench.max_over_ranks(10.0 * (r + 1), w)
    sm = bench.sum_over_ranks(float(r + 1), w)

    class A:
        steps, warmup, workload = 1, 1, "none"
    ref = bench.run_reference(A, r, w) if r == 1 else "skip"
    q.put((r, w, dist.get_backend(), mx, sm, ref))
    bench.barrier(w)
    dist.destroy_process_group()


def test_two_host_ranks_reduce_and_only_rank0_runs_reference():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, (rank, w, backend, mx, sm, ref) in enumerate(out):
        assert rank == r and w == world and backend == "gloo"
        assert mx == 20.0 and sm == 3.0
    assert out[1][5] is None   # rank 1 does no reference work
