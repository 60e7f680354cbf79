"""The multi-rank plumbing of bench.py on CPU: two gloo ranks, spawned as processes.

The forward has no exchange step, so N GPUs run N replicas; what the ranks share is a barrier,
the maximum of their device times and the teardown (bench.RankGroup), and the whole-job value
is all ranks' units over the slowest rank's time (bench.aggregate).  A rank that raises before
its reduction ends the other rank's collective with an error instead of a hang."""
import multiprocessing as mp
import os
import socket
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, mode, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    try:
        g = bench.RankGroup("gloo", timeout_s=10)
        g.barrier()
        if mode == "raise" and rank == 1:
            raise RuntimeError("rank 1 fails before its reduction")
        ms = g.max(100.0 + 25.0 * rank)            # this rank's device time for the timed steps
        g.close()
        q.put((rank, "ok", ms, bench.aggregate(11.0, world, ms)))
    except Exception as e:                           # reported to the test, which decides
        q.put((rank, "error", type(e).__name__, str(e)[:200]))


def _run(mode, world=2, limit=90):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, mode, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(limit)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
    res = {}
    while not q.empty():
        r = q.get()
        res[r[0]] = r[1:]
    return res, alive


def test_two_ranks_reduce_the_slowest_time():
    res, alive = _run("ok")
    assert not alive
    assert res[0][0] == "ok" and res[1][0] == "ok", res
    assert res[0][1] == res[1][1] == 125.0                   # the max over ranks, on every rank
    assert abs(res[0][2] - 2 * 11.0 / 0.125) < 1e-9          # both ranks' audio over the slowest time


def test_a_failing_rank_ends_the_others_collective():
    res, alive = _run("raise")
    assert not alive                                          # nobody waits for good
    assert res[1][0] == "error" and res[1][1] == "RuntimeError"
    assert res[0][0] == "error", res                          # rank 0's reduction fails instead of hanging


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    env = {k: os.environ.pop(k) for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK") if k in os.environ}
    try:
        g = bench.RankGroup("gloo")
        assert g.world == 1 and g.max(3.5) == 3.5
        g.barrier()
        g.close()
    finally:
        os.environ.update(env)
