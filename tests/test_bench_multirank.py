"""The benchmark's multi-rank host logic on CPU: two gloo ranks (no GPU).

On a multi-GPU node bench.py runs one rank per GPU over NCCL; the parts that decide
the reported number -- the max over ranks of every timing, the whole-job
throughput, and which rank prints -- do not depend on the backend and are
exercised here with gloo."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        slowest = bench.max_over_ranks(10.0 + 5.0 * rank)      # rank 1 is slower
        q.put((rank, slowest))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got == {0: 15.0, 1: 15.0}


def test_max_over_ranks_without_group():
    assert bench.max_over_ranks(3.5) == 3.5


def test_job_throughput_is_weak_scaling():
    # 2 ranks, 504,375,808 bytes each per step, 0.1 ms per step -> 2 x 5043.76 GB/s
    assert bench.job_throughput(2, 504_375_808, 1e-4) == pytest.approx(10087.51616)
    assert bench.job_throughput(1, 10**9, 1.0) == 1.0


def test_reference_arm_runs_on_rank_zero_only():
    args = type("A", (), dict(workload="fp32_256x768", steps=1, warmup=0))()
    assert bench.run_reference(args, world=2, rank=1) is None
    line = bench.run_reference(args, world=1, rank=0)
    assert line["impl"] == "reference" and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["unit"] == "GB/s" and line["value"] > 0


def test_source_hash_ignores_comments_only():
    """The traffic figure's key: comment edits keep it, code edits change it,
    and string literals (inline PTX) survive comment stripping."""
    a = 'asm("mov.u32 %0, 1; // not a comment");  // comment\nint x = 2; /* c */\n'
    b = 'asm("mov.u32 %0, 1; // not a comment");  // other words\n\nint x = 2;\n'
    c = 'asm("mov.u32 %0, 1; // not a comment");\nint x = 3;\n'
    assert bench.strip_comments(a) == bench.strip_comments(b)
    assert bench.strip_comments(a) != bench.strip_comments(c)
    assert "// not a comment" in bench.strip_comments(a)
    assert len(bench.source_sha256()) == 64
