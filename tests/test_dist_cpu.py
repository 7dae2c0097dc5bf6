"""The N > 1 host path of bench.py on CPU: two gloo ranks, the max-over-ranks timing
reduction, the barrier, the rank environment and the weak-scaling aggregate."""
import os
import tempfile

import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rendezvous():
    """A fresh file for the ranks to meet through (no TCP port to race for)."""
    fd, path = tempfile.mkstemp(prefix="gloo_rdzv_")
    os.close(fd)
    os.unlink(path)
    return "file://" + path


def _worker(rank, world, init, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from datetime import timedelta
    dist.init_process_group("gloo", init_method=init, rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    w, r, l = bench.dist_env()
    t = bench.max_over_ranks(10.0 + 5.0 * rank, w)
    bench.barrier(w)
    out.put((r, w, l, t))
    dist.destroy_process_group()


def test_two_gloo_ranks_reduce_max_and_agree():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    init = _rendezvous()
    procs = [ctx.Process(target=_worker, args=(r, 2, init, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [x[0] for x in res] == [0, 1]
    assert all(x[1] == 2 for x in res)
    assert [x[2] for x in res] == [0, 1]
    assert all(x[3] == 15.0 for x in res)  # every rank sees the slowest rank's time


def test_single_process_paths_and_aggregate():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    bench.barrier(1)
    # N ranks, each its own batch: N x the work over the slowest rank's time
    one = bench.aggregate_tflops(1, 8.42e11, 1.4)
    assert abs(bench.aggregate_tflops(4, 8.42e11, 1.4) - 4 * one) < 1e-9
    assert abs(one - 8.42e11 / 1.4e-3 / 1e12) < 1e-9


def _worker_one_dies(rank, world, init, out, passed):
    """Rank 1 leaves between steps (after the group formed, before the next
    collective); rank 0's next collective must end with an error, not wait.
    Rank 1 leaves only once rank 0 has come out of the barrier (`passed`), so
    that the collective that meets the missing rank is the next one."""
    import sys
    import time
    sys.path.insert(0, ROOT)
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from datetime import timedelta
    dist.init_process_group("gloo", init_method=init, rank=rank, world_size=world, timeout=timedelta(seconds=10))
    import bench
    bench.barrier(world)                      # both ranks reach the first step
    if rank == 1:
        passed.wait(60)
        os._exit(0)                            # leaves with nothing in flight
    passed.set()
    time.sleep(0.5)                            # rank 1 is gone before the next collective
    t0 = time.time()
    try:
        bench.max_over_ranks(1.0, world)
        out.put(("no error", time.time() - t0))
    except Exception as e:                     # gloo reports the lost peer
        out.put((type(e).__name__, time.time() - t0))
    # a queue hands its items to a feeder thread: flush it before the hard exit
    out.close()
    out.join_thread()
    os._exit(0)


def test_a_rank_that_leaves_ends_the_next_collective_with_an_error():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    init = _rendezvous()
    passed = ctx.Event()
    procs = [ctx.Process(target=_worker_one_dies, args=(r, 2, init, q, passed)) for r in range(2)]
    for p in procs:
        p.start()
    kind, secs = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
    assert kind != "no error"
    assert secs < 30.0                         # bounded by the group's 10 s timeout, not a hang
