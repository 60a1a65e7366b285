"""Host logic of the multi-rank benchmark on CPU: two gloo ranks, the way
`torchrun --nproc-per-node 2 bench.py` starts them (RANK / WORLD_SIZE /
MASTER_* in the environment).  Timings are combined as the max over ranks,
the value counts every rank's units, and a rank that never joins a
collective makes the other rank's collective fail within its timeout instead
of hanging."""
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, mode, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    try:
        import bench
        d = bench.Dist(backend="gloo", timeout_s=4.0 if mode == "drop" else 60.0)
        my_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        d.barrier()
        if mode == "drop" and rank == 1:
            q.put((rank, "left"))  # leaves between steps, before the timing collective
            return
        try:
            worst = d.max(my_ms)
        except Exception as e:  # the collective gives up instead of hanging
            q.put((rank, "error:" + type(e).__name__))
            return
        value = bench.job_rate(d.world, 1000.0, 4, worst)
        d.barrier()
        d.close()
        q.put((rank, (worst, value)))
    except Exception as e:  # report instead of hanging the parent
        q.put((rank, "exc:" + repr(e)))


def _run(mode, world=2, timeout=90):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, mode, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    try:
        for _ in range(world):
            r, v = q.get(timeout=timeout)
            out[r] = v
    finally:
        for p in procs:
            p.join(timeout=30)
            if p.is_alive():
                p.kill()
    return out


def test_max_over_ranks_and_whole_job_value():
    out = _run("ok")
    assert set(out) == {0, 1}
    for r in (0, 1):
        worst, value = out[r]
        assert worst == 15.0  # the slower rank's time, on every rank
        assert value == pytest.approx(2 * 1000.0 * 4 / 15e-3)  # both ranks' units


def test_rank_that_leaves_makes_the_collective_fail_not_hang():
    out = _run("drop")
    assert out[1] == "left"
    assert isinstance(out[0], str) and out[0].startswith(("error:", "exc:")), out[0]


def test_job_rate_single_rank():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.job_rate(1, 33.29e9, 10, 1000.0) == pytest.approx(33.29e10)
