"""The bench's multi-rank logic on CPU: two gloo ranks (no GPU).

Each rank reports a different device time; both must see the maximum, and the
whole-job rate counts every rank's tokens over the slowest rank's time.  The
reference arm runs on rank 0 only: any other rank returns without work.
"""
import os
import socket
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(dist, 10.0 + 5.0 * rank, "cpu")  # rank 1 is the slow one
        rate = bench.whole_job_rate(world, 105, 20, ms / 1e3)
        dist.barrier()
    finally:
        dist.destroy_process_group()
    # the reference arm: only rank 0 runs the oracle
    os.environ["RANK"] = str(rank)
    ran = None
    if rank != 0:
        ran = bench.run_reference(None, None, None, None, None, None)
    out.put((rank, ms, rate, ran))


def test_two_gloo_ranks_agree_on_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = {}
    for _ in procs:
        rank, ms, rate, ran = q.get(timeout=120)
        got[rank] = (ms, rate, ran)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got[0][0] == got[1][0] == 15.0
    assert got[0][1] == got[1][1] == pytest.approx(2 * 105 * 20 / 0.015)
    assert got[1][2] is None


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(None, 3.5, "cpu") == 3.5
    assert bench.whole_job_rate(1, 105, 50, 0.1) == pytest.approx(52500.0)


def test_parity_stats_are_the_tolerance_figures():
    import numpy as np
    import bench
    want = np.array([[3.0, -4.0], [0.0, 5.0]])  # RMS = sqrt(50 / 4)
    got = want + np.array([[0.5, 0.0], [0.0, -0.25]])
    mx, l1 = bench.parity_stats(got, want)
    assert np.isclose(mx, 0.5 / np.sqrt(12.5))
    assert np.isclose(l1, 0.75 / 12.0)
    assert bench.parity_stats(want, want) == (0.0, 0.0)
