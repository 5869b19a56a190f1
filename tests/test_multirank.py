"""The multi-rank (torchrun, N > 1) host logic of bench.py on CPU with two gloo ranks.

With N GPUs every rank runs an independent seeded batch (data-parallel
replicas, no collective on the data path); the job's time is the slowest
rank's, and the job's throughput counts the work of all ranks."""
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


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import workloads

        seed = bench.rank_seed(0, rank)
        lens = workloads.doc_lengths(workloads.WORKLOADS["llama32_1b_32k"], seed)
        elapsed = 100.0 + 25.0 * rank  # pretend per-rank device times
        job = bench.max_over_ranks(elapsed, dist, "cpu")
        out.put((rank, seed, tuple(lens), job, bench.job_throughput(1e12, 10, world, job)))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_ranks_replicas_and_max_time():
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
    (r0, s0, l0, j0, v0), (r1, s1, l1, j1, v1) = res
    assert (s0, s1) == (0, 1)            # each rank its own batch
    assert l0 != l1                      # ... so the document mixes differ
    assert j0 == j1 == 125.0             # the job time is the slowest rank's
    assert v0 == v1 == pytest.approx(2 * 1e12 * 10 / 0.125 / 1e12)  # all ranks' work over that time


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.5, None) == 7.5
    assert bench.job_throughput(2e12, 5, 1, 1000.0) == pytest.approx(10.0)
