"""The multi-process plumbing of bench.py on CPU: two gloo ranks.

bench.py runs one replica of the decode stack per GPU (no data-path
collective); across ranks it only takes the slowest rank's time and sums the
bytes of all ranks. These tests run that logic with world_size 2 on gloo.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    from datetime import timedelta
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=60))
    try:
        ms = [3.0, 5.0][rank]                      # rank 1 is the slower one
        worst = bench.max_over_ranks(ms, "cpu")
        value = bench.whole_job_gbs(world, 1_000_000_000, worst)
        out.put((rank, worst, value))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank_and_sum_bytes():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(out.get(timeout=5) for _ in range(2))
    for rank, worst, value in res:
        assert worst == pytest.approx(5.0)
        # 2 ranks x 1 GB in 5 ms = 400 GB/s
        assert value == pytest.approx(400.0)


def test_single_process_needs_no_process_group():
    assert bench.max_over_ranks(2.5, "cpu") == 2.5
    assert bench.whole_job_gbs(1, 2_000_000_000, 1.0) == pytest.approx(2000.0)


def test_reference_arm_other_ranks_exit_without_work(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class Args:
        steps, warmup, gpus, layers = 1, 0, 2, 32
    assert bench.run_reference(Args()) == 0
