"""The multi-rank plumbing of bench.py on CPU: two gloo ranks.

bench.py shards the work as independent replicas (each rank runs its own
sequences, no data-path collective); the only cross-rank steps are the
barriers around the timed region and the maximum of the per-rank device
times, from which the whole-job throughput is computed.  These run here as
two spawned processes over gloo on 127.0.0.1.
"""
import datetime
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    torch.distributed.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        w, r, _ = bench.dist_setup()
        bench.barrier(w)
        ms = bench.max_over_ranks(times[r], w)
        value = bench.job_throughput(1000, 4, ms, w)
        bench.barrier(w)
        q.put((r, w, ms, value))
    finally:
        torch.distributed.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port, world, times = _free_port(), 2, [3.0, 5.0]
    procs = [ctx.Process(target=_worker, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=90) for _ in range(world))
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    assert [o[0] for o in out] == [0, 1]
    for _, w, ms, value in out:
        assert w == 2
        assert ms == 5.0                                 # max over ranks, not the local time
        assert value == pytest.approx(2 * 1000 * 4 / 5e-3)   # units of all ranks / slowest time


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.5, 1) == 2.5
    assert bench.job_throughput(10, 2, 4.0, 1) == pytest.approx(5000.0)


def test_recorded_traffic_is_keyed_by_code_not_comments(tmp_path):
    """bench.py uses a committed ncu traffic figure only for the code it was
    taken on: a comment-only edit keeps the key, a code edit changes it."""
    sys.path.insert(0, ROOT)
    import bench
    code = "int f(int x) {\n  // one comment\n  return x + 1; /* another */\n}\n"
    assert bench._code_only(code) == bench._code_only(code.replace("one comment", "reworded comment"))
    assert bench._code_only(code) != bench._code_only(code.replace("x + 1", "x + 2"))
    assert "comment" not in bench._code_only(code)
    # every kernel named in the traffic table has a current key or is ignored
    for line in open(os.path.join(ROOT, "profiles", "ncu_traffic.txt")):
        f = line.split()
        if line.startswith("#") or len(f) < 4:
            continue
        got = bench.recorded_traffic(f[0], f[1])
        assert got is None or got == float(f[3])
