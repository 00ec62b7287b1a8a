"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The decode path shards by request: each rank owns its requests and there is
no collective on the data path.  What the ranks do share is the timing
protocol: per-rank device timings combine as a maximum over ranks, the job's
rate counts every rank's queries, and only rank 0 prints."""
import contextlib
import io
import os
import socket
import sys
from datetime import timedelta

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, ws, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    from compressed_sparse_long_hca_b200 import inputs as I
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=timedelta(seconds=60))
    try:
        vals = bench.max_over_ranks([1.0 + rank, 5.0 - rank, 2.5 * rank], ws, "cpu")
        seeds = [None] * ws
        dist.all_gather_object(seeds, bench.rank_seed(I.C4, rank))
        q.put((rank, vals, seeds))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_and_disjoint_requests():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = [q.get(timeout=120) for _ in ps]
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, vals, seeds in res:
        assert vals == [2.0, 5.0, 2.5], f"rank {rank}: {vals}"
        assert len(set(seeds)) == 2, "ranks must own disjoint requests"


def test_whole_job_rate_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    # 2 ranks x 4 queries x 10 steps in 5 ms (the slowest rank)
    assert bench.whole_job_rate(2, 4, 10, 5.0) == pytest.approx(16000.0)
    assert bench.whole_job_rate(1, 4, 10, 5.0) == pytest.approx(8000.0)


def test_reference_arm_only_rank0_prints(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class Args:
        workload, steps, warmup = "tiny-csa", 1, 3

    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(Args())
    assert buf.getvalue() == ""
