"""The multi-rank plumbing of bench.py, run as two gloo ranks on the CPU.

With --gpus N the benchmark runs one process per GPU: every rank processes its own
copy of the work, the timings meet in a max over ranks, the whole-job value is the
work of all ranks over the slowest rank's time, and only rank 0 prints.  The decode
path itself has no data-path collective (independent problems), so these are the only
collective steps there are.  The same helpers run here on a gloo process group.
"""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank, world, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))


def _timing_worker(rank, world, port, q):
    try:
        if ROOT not in sys.path:
            sys.path.insert(0, ROOT)
        _env(rank, world, port)
        import torch.distributed as dist

        import bench
        w, r, local = bench._dist_setup(world, backend="gloo")
        ms = 2.0 + 3.0 * r                     # rank 1 is the slow one
        m = bench._max_over_ranks(w, ms, device="cpu")
        bench._barrier(w, cuda=False)
        v = bench.aggregate_gbs(w, 1_000_000, 10, m)
        q.put(("ok", r, w, local, m, v))
        dist.destroy_process_group()
    except Exception as e:                     # reported to the parent, never hangs it
        q.put(("err", rank, repr(e)))


def _spawn(target, world, extra=()):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, q, *extra)) for r in range(world)]
    for p in procs:
        p.start()
    out = []
    try:
        for _ in range(world):
            out.append(q.get(timeout=120))
    finally:
        for p in procs:
            p.join(timeout=30)
            if p.is_alive():
                p.kill()
    return out


def test_two_ranks_take_the_slowest_time_and_sum_the_work():
    res = _spawn(_timing_worker, 2)
    assert all(r[0] == "ok" for r in res), res
    by_rank = {r[1]: r for r in res}
    assert set(by_rank) == {0, 1}
    for rank, (_, r, w, local, m, v) in by_rank.items():
        assert w == 2 and local == rank
        assert m == 5.0                         # max(2.0, 5.0) on both ranks
        # 2 ranks x 1e6 bytes x 10 steps over 5 ms = 4 GB/s
        assert v == pytest.approx(4.0)


def test_single_rank_needs_no_process_group(monkeypatch):
    import bench
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    world, rank, local = bench._dist_setup(1, backend="gloo")
    assert (world, rank, local) == (1, 0, 0)
    assert bench._max_over_ranks(world, 3.5, device="cpu") == 3.5
    assert bench.aggregate_gbs(1, 2_000_000, 4, 1.0) == pytest.approx(8.0)


class _Args:
    steps = 2
    warmup = 0


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    """Under torchrun the reference arm (the oracle on the host) is run and printed by
    rank 0 alone; the other ranks return without work or output."""
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    buf = io.StringIO()
    with redirect_stdout(buf):
        assert bench.run_reference(_Args()) is None
    assert buf.getvalue() == ""

    monkeypatch.setenv("RANK", "0")
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(_Args())
    lines = [l for l in buf.getvalue().splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["steps"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
