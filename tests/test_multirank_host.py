"""World-size-2 gloo run of the benchmark's multi-rank plumbing on CPU: each rank is an
independent replica, timings reduce by max, and the job throughput adds the ranks' units."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import dsa_inputs as DI
        # replicas draw their own inputs (seed = rank) of the same shapes
        inp = DI.make_inputs("tiny_decode", seed=rank, with_mla=False)
        units = bench.work_units(inp)
        t = [0.5 + rank, 2.0 - rank]                     # per-rank seconds (device, e2e)
        tmax = bench.max_over_ranks(t, world, "cpu")
        v = bench.weak_scaling_value(units["pairs"], 10, world, tmax[0])
        q.put((rank, tmax, v, units["pairs"], float(inp.idx_q[0, 0, 0, 0])))
    finally:
        dist.destroy_process_group()


def test_two_rank_weak_scaling_plumbing():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    (r0, t0, v0, u0, x0), (r1, t1, v1, u1, x1) = res
    assert t0 == t1 == [1.5, 2.0]                        # max over ranks, seen by both
    assert u0 == u1 == 1024                              # same shapes on every replica
    assert x0 != x1                                      # but independent data
    assert v0 == pytest.approx(1024 * 10 * 2 / 1.5)


def _failing_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import time
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        # the failing rank: leaves between steps, before the timing reduction, without a collective
        raise SystemExit(3)
    import bench
    t0 = time.time()
    try:
        bench.max_over_ranks([1.0, 2.0], world, "cpu")
        q.put(("no error", time.time() - t0))
    except Exception as e:                               # the lost peer surfaces as an error
        q.put((type(e).__name__, time.time() - t0))
    finally:
        try:
            dist.destroy_process_group()
        except Exception:
            pass


def test_a_lost_rank_ends_the_reduction_with_an_error():
    """Failure detection on the host: when a rank leaves, the surviving rank's max-over-ranks
    reduction ends with an error (the process group's short timeout or the closed connection)
    instead of waiting for ever."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_failing_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert procs[1].exitcode == 3
    what, waited = q.get(timeout=5)
    assert what != "no error"
    assert waited < 60
