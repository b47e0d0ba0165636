"""The replica plumbing of bench.py across two processes on CPU (gloo backend): joining the
process group, the barrier around the timed region, the maximum over ranks of the device time,
the whole-job throughput, and teardown.  Each rank runs an independent replica of the layer (no
data-path collective), so these host steps are the whole multi-rank path."""
import multiprocessing as mp
import os
import socket

import pytest


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    w, r, _ = bench.dist_setup(world)
    bench.ranks_init(w, "gloo", timeout_s=60)
    bench.ranks_barrier(w)
    ms = bench.ranks_max(times[r], w)
    value = bench.job_throughput(64 * 10, w, ms)
    bench.ranks_finish(w)
    q.put((r, w, ms, value))


def test_two_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    times = [12.5, 20.0]                      # rank 1 is the slow one
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, times, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        res = sorted(q.get(timeout=120) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
    assert [p.exitcode for p in procs] == [0, 0]
    for r, (rank, world, ms, value) in enumerate(res):
        assert (rank, world) == (r, 2)
        assert ms == 20.0                     # every rank sees the slowest rank's time
        assert value == pytest.approx(2 * 64 * 10 / 0.020)   # both ranks' tokens over it


def test_single_rank_needs_no_group():
    import bench
    assert bench.ranks_max(3.25, 1) == 3.25
    assert bench.job_throughput(64 * 10, 1, 20.0) == pytest.approx(64 * 10 / 0.020)
    bench.ranks_init(1)                       # no process group for one rank
    bench.ranks_barrier(1)
    bench.ranks_finish(1)


def test_reference_arm_runs_on_rank_zero_only():
    import bench
    # a non-zero rank returns before touching its arguments or the oracle
    assert bench.reference(None, 2, 1) is None
