"""Multi-process path of the benchmark on CPU: two ranks over gloo.

The benchmark runs one replica per rank (the (batch, kv head) problems are
independent, so there is no data-path collective); the only cross-rank steps
are the barriers around the timed region and the max over ranks of the
measured times.  These run here with world size 2 on the host."""
import os
import socket

import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch.distributed as dist
    import bench
    r, w, local = bench.dist_setup()
    assert (r, w, local) == (rank, world, rank)
    assert dist.get_backend() == "gloo"
    bench.barrier(w)
    # every rank reports its own time; all of them see the slowest
    m = bench.dist_max(1.5 + 2.0 * rank, w)
    bench.barrier(w)
    out.put((rank, m))
    dist.destroy_process_group()


def test_two_ranks_barrier_and_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert results == {0: 3.5, 1: 3.5}


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.dist_max(2.25, 1) == 2.25
    bench.barrier(1)   # no-op without a process group
