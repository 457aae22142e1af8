"""The N > 1 path of the benchmark on CPU: two ranks over gloo.

With N GPUs every rank runs an independent replica of the step (the method
shards by replica: no collective on the data path).  What the ranks share is
the host logic: the launcher's environment, the max over ranks of each
rank's time, and the whole-job rate.  These tests run that logic in two
processes on 127.0.0.1 with the gloo backend.
"""

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, ms_by_rank, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import datetime
    w, r, local = bench.dist_env()
    dist.init_process_group("gloo", rank=r, world_size=w, timeout=datetime.timedelta(seconds=60))
    try:
        dev = torch.device("cpu")
        ms = bench.max_over_ranks(ms_by_rank[r], dev, w)
        flops = bench.train_flops(bench.M, bench.D, bench.D, bench.R)
        value = bench.job_rate(w, flops, ms) / 1e12
        dist.barrier()
        out.put((r, w, local, ms, value))
    finally:
        dist.destroy_process_group()


def _run(ms_by_rank):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(i, WORLD, port, ms_by_rank, out)) for i in range(WORLD)]
    for p in procs:
        p.start()
    res = [out.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(res)


def test_dist_env_defaults(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.dist_env() == (1, 0, 0)
    monkeypatch.setenv("WORLD_SIZE", "8")
    monkeypatch.setenv("RANK", "5")
    monkeypatch.setenv("LOCAL_RANK", "5")
    assert bench.dist_env() == (8, 5, 5)


def test_single_rank_needs_no_process_group():
    assert not dist.is_initialized()
    assert bench.max_over_ranks(0.25, torch.device("cpu"), 1) == 0.25


def test_job_rate_weak_scaling():
    # every rank did the same work; the slowest rank's time sets the rate
    assert bench.job_rate(1, 1e12, 1000.0) == pytest.approx(1e12)
    assert bench.job_rate(4, 1e12, 500.0) == pytest.approx(8e12)


def test_two_ranks_take_the_max_time():
    ms_by_rank = [0.170, 0.185]
    res = _run(ms_by_rank)
    flops = bench.train_flops(bench.M, bench.D, bench.D, bench.R)
    for i, (rank, world, local, ms, value) in enumerate(res):
        assert (rank, world, local) == (i, WORLD, i)
        assert ms == max(ms_by_rank)
        # whole-job value: the units both ranks processed over the slowest time
        assert value == pytest.approx(WORLD * flops / (max(ms_by_rank) * 1e-3) / 1e12)


def test_two_ranks_agree_when_the_slow_rank_is_rank_0():
    res = _run([2.0, 1.0])
    assert [r[3] for r in res] == [2.0, 2.0]
    assert res[0][4] == res[1][4]


def test_reference_arm_runs_on_rank_0_only(monkeypatch, capsys):
    """Under a launcher with N > 1 the CPU reference arm prints one line on
    rank 0; the other ranks return at once, without work or output."""
    import types
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("LOCAL_RANK", "1")
    args = types.SimpleNamespace(quick=True, steps=1, warmup=0, gpus=2)
    assert bench.run_reference(args) is None
    assert capsys.readouterr().out == ""
