"""The N > 1 bench path on CPU: two gloo ranks, no GPU.  Checks that the
timing reduction takes the slowest rank, that whole-job throughput counts
every rank's bytes over that time, and that the reference arm runs on rank
0 only (other ranks exit 0 without work)."""
import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    ms = bench.max_over_ranks(10.0 + 5.0 * rank, world)  # rank 1 is slower
    gbs = bench.job_throughput(1_000_000_000, world, 4, ms)
    bench.barrier(world)
    # the reference arm: rank 0 prints, the others return 0 at once
    class A:
        steps, warmup = 1, 0
    rc = bench.run_reference(A) if rank != 0 else 0
    q.put((rank, ms, gbs, rc))
    dist.destroy_process_group()


def test_two_gloo_ranks_reduce_time_and_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, gbs, rc in res:
        assert ms == pytest.approx(15.0)            # max over ranks
        assert gbs == pytest.approx(2 * 4 * 1e9 / 15e-3 / 1e9)
        assert rc == 0
