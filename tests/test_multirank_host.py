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


def test_gpus_flag_starts_one_rank_per_gpu():
    """`bench.py --gpus N` outside a launcher re-executes itself as N ranks under
    torch.distributed.run (rendezvous on 127.0.0.1); checked with the reference arm, which needs
    no GPU: rank 0 prints the line with n_gpus = N."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--workload", "tiny_decode", "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, timeout=600, env=env, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1 and lines[0]["n_gpus"] == 2 and lines[0]["impl"] == "reference"


def test_gpus_flag_must_match_the_launched_world():
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2", "--workload", "tiny_decode"],
                       capture_output=True, text=True, timeout=300, env=env, cwd=root)
    assert r.returncode == 2 and "WORLD_SIZE=1" in r.stderr


def _head_parallel_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import numpy as np
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import importlib.util
        root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
        spec = importlib.util.spec_from_file_location(
            "head_parallel", os.path.join(root, "sparse_attention_keys_b200", "head_parallel.py"))
        hp = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(hp)            # the plumbing alone: no CUDA library on this host
        import dsa_inputs as DI
        from oracle import dsa_oracle as O
        inp = DI.make_custom(2, 2, 96, 16, decode=False, seed=11)    # identical inputs on every rank
        # only the source rank has the indexer's selection; the others hold garbage until the broadcast
        if rank == 0:
            rng = np.random.default_rng(5)
            idx_np = np.stack([np.stack([np.sort(rng.choice(96, 16, replace=False)) for _ in range(2)])
                               for _ in range(2)]).astype(np.int32)
        else:
            idx_np = np.full((2, 2, 16), 12345, np.int32)
        idx = torch.from_numpy(idx_np.copy())
        sl = hp.head_shard(rank, world)

        def oracle_attend(q_local, kv, idx_t):
            return O.sparse_mla(q_local, kv, idx_t.numpy())

        out, lse = hp.sparse_mla_head_parallel(np.ascontiguousarray(inp.mla_q[:, :, sl]), inp.mla_kv, idx,
                                               attend=oracle_attend)
        q.put((rank, sl.start, sl.stop, idx.numpy().copy(), out, lse))
    finally:
        dist.destroy_process_group()


def test_head_parallel_plumbing_two_ranks():
    """Two gloo ranks: rank 0's selected indices reach rank 1 through the broadcast, each rank
    attends with its 64 heads (the oracle stands in for the kernel on CPU), and the two shards
    put together are the 128-head result."""
    import numpy as np
    import dsa_inputs as DI
    from oracle import dsa_oracle as O
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_head_parallel_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted([q.get(timeout=300) for _ in range(2)], key=lambda x: x[0])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    (r0, a0, b0, idx0, out0, lse0), (r1, a1, b1, idx1, out1, lse1) = res
    assert (a0, b0, a1, b1) == (0, 64, 64, 128)
    assert np.array_equal(idx0, idx1) and not np.any(idx1 == 12345)
    inp = DI.make_custom(2, 2, 96, 16, decode=False, seed=11)
    full, full_lse = O.sparse_mla(inp.mla_q, inp.mla_kv, idx0)
    assert np.array_equal(np.concatenate([out0, out1], axis=2), full)
    assert np.array_equal(np.concatenate([lse0, lse1], axis=2), full_lse)
