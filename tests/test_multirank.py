"""The benchmark's multi-rank plumbing on CPU ranks over gloo (world size 2):
barrier, the max of the ranks' step times, the weak-scaling aggregate, and
the reference arm running on rank 0 alone."""
import os
import socket

import pytest
import torch.multiprocessing as tmp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    import bench
    d = bench.Dist(backend="gloo")
    d.barrier()
    my_ms = 1.5 + rank            # rank 1 is the slow one
    worst = d.max(my_ms)
    value = bench.weak_scaling_value(16, d.world, worst)
    q.put((rank, d.world, worst, value))
    d.close()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    port = _free_port()
    ctx = tmp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, world, worst, value in out:
        assert world == 2 and worst == 2.5
        assert value == pytest.approx(16 * 2 / 2.5e-3)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    class A:
        steps, warmup, seed = 1, 1, 0
    assert bench.run_reference(A(), bench.workloads.CONFIGS["tiny"]) == 0


def _failing_rank_main(rank, world, port, q, mode):
    import sys
    import time
    sys.path.insert(0, ROOT)
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    import bench
    d = bench.Dist(backend="gloo", timeout_s=5)
    if rank == 1:
        if mode == "exit":
            os._exit(0)                  # dies between steps, with nothing in flight
        time.sleep(60)                   # alive but never reaches the barrier
        return
    t0 = time.time()
    try:
        d.barrier()
        d.max(1.0)
        q.put(("no error", time.time() - t0))
    except Exception as e:              # the surviving rank learns of it on the host
        q.put((type(e).__name__, time.time() - t0))


@pytest.mark.parametrize("mode", ["exit", "silent"])
def test_a_lost_rank_ends_the_others_collectives_with_an_error(mode):
    """A rank that exits, or that stops answering, makes the other rank's next
    collective raise within the process group's timeout instead of waiting for
    good (host-side failure detection; no GPU involved)."""
    port = _free_port()
    ctx = tmp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_failing_rank_main, args=(r, 2, port, q, mode)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        what, waited = q.get(timeout=90)
    finally:
        for p in procs:
            if p.is_alive():
                p.terminate()
            p.join(timeout=30)
    assert what != "no error"
    assert waited < 60
