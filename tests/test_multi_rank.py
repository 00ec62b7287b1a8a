"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The decode path shards by request: each rank owns its requests and there is
no collective on the data path.  What the ranks do share is the timing
protocol: per-rank device timings combine as a maximum over ranks, the job's
rate counts every rank's queries, and only rank 0 prints."""
import contextlib
import io
import json
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


def test_reference_arm_line_keeps_the_contract(monkeypatch):
    """Rank 0 of the reference arm (the oracle on the host cores) prints one
    JSON line with the contract's keys, the same metric and unit as the
    CUDA arm, and its own cpu_baseline and e2e objects."""
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")

    class Args:
        workload, steps, warmup = "tiny-csa", 1, 3

    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(Args())
    lines = [x for x in buf.getvalue().splitlines() if x.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["unit"] == bench.UNIT and d["higher_is_better"] is True
    assert d["config"]["workload"] == "tiny-csa" and d["steps"] == 1 and d["warmup"] == 3
    assert d["value"] > 0 and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_bench_byte_counts_and_rooflines():
    """Algorithmic bytes per stored key / row, and the two rooflines from a
    made-up timing: 1 ms per step and per launch."""
    import bench
    from compressed_sparse_long_hca_b200 import inputs as I
    assert bench.key_bytes(I.C4, "mixed") == 68          # 64 B E2M1 codes + 4 E8M0 scales
    assert bench.row_bytes(I.C4, "mixed") == 580         # 448 E4M3 + 64 BF16 + fp32 scale
    assert bench.key_bytes(I.C1, "f32") == 128 and bench.row_bytes(I.C1, "f32") == 256
    assert bench.workload_fmt(I.C1) == "f32" and bench.workload_fmt(I.C4) == "mixed"
    m = {"t_mid": 1 << 20, "idx_ms": 1.0, "step_ms": 1.0}
    r = bench.rooflines(I.C4, m, steps=1)
    keys = 4 * ((1 << 18) * 68 + 64 * 128 * 4 + 64 * 4)
    assert r["roofline"]["algorithmic_bytes_per_launch"] == keys
    assert r["roofline"]["achieved"] == pytest.approx(keys / 1e-3 / 1e9)
    rows = 4 * ((1024 + 128) * 580 + 2 * 128 * 512 * 2)
    assert r["step_roofline"]["algorithmic_bytes_per_step"] == keys + rows
    h = bench.rooflines(I.C5_HCA_1M, m, steps=1)
    assert h["roofline"]["bound"] == "tensor"
    assert h["roofline"]["algorithmic_flops_per_launch"] == 4 * 4.0 * 128 * (8192 + 128) * 512
