"""The bench's multi-rank logic on CPU, world size 2 over gloo: each rank runs its own
replica (own seed), the reported time is the slowest rank's, the whole-job value counts
every rank's work, and the reference arm prints from rank 0 only."""
import importlib.util
import io
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        b = _bench()
        t_local = [0.25, 0.75][rank]                      # rank 1 is the slow one
        t_max = b.max_over_ranks(t_local, world, "cpu")
        w = b.rank_workload(b.WORKLOADS["small-h2-n1024"], rank)
        out.put((rank, t_max, w.seed))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_distinct_seeds():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [0.75, 0.75]
    assert res[0][2] != res[1][2]


def test_whole_job_value_counts_every_rank():
    b = _bench()
    assert b.whole_job_tops(2e12, 1, 0.5) == pytest.approx(4.0)
    assert b.whole_job_tops(2e12, 4, 0.5) == pytest.approx(16.0)
    assert b.max_over_ranks(0.3, 1) == 0.3


def test_reference_arm_prints_from_rank_zero_only(monkeypatch):
    b = _bench()
    monkeypatch.setenv("RANK", "1")

    class Args:
        oracle_rows, warmup, steps, gpus = 4, 1, 1, 2

    buf = io.StringIO()
    with redirect_stdout(buf):
        assert b.run_reference(Args(), b.WORKLOADS["small-h2-n1024"]) == 0
    assert buf.getvalue() == ""
