"""The multi-rank path of bench.py (independent replicas, one per GPU) on
CPU ranks over gloo: the time is the maximum over ranks, the throughput
counts every rank's tokens, and the reference arm runs on rank 0 only."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        r, lr, w = bench.env_rank()
        ms = 10.0 + 5.0 * rank                      # rank 1 is the slow one
        ms_max = bench.max_over_ranks(ms, w, "cpu")
        out.put((r, lr, w, ms_max, bench.job_tokens_per_s(w, 256, ms_max)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank_and_count_all_tokens():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, (r, lr, w, ms_max, v) in enumerate(res):
        assert (r, lr, w) == (rank, rank, 2)
        assert ms_max == 15.0
        assert v == pytest.approx(2 * 256 / 0.015)


def test_one_rank_needs_no_process_group():
    assert bench.max_over_ranks(12.5, 1, "cpu") == 12.5
    assert bench.job_tokens_per_s(1, 256, 100.0) == pytest.approx(2560.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--gpus", "2"])
    bench.run_reference(bench.parse())
    assert capsys.readouterr().out == ""
