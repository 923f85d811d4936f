"""bench.py's multi-rank plumbing on CPU: two gloo ranks, one process each, set up the way torchrun sets
them up (RANK / WORLD_SIZE / MASTER_* over 127.0.0.1): rendezvous, max-over-ranks timing, the whole-job
rate of weak scaling, and the reference arm that only rank 0 runs."""
import importlib.util
import os
import socket
import time

import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_multirank_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    b = _bench()
    r, w = b.dist_init(world, backend="gloo")
    ms = b.max_over_ranks(10.0 + 5.0 * r, w, "cpu")          # rank 1 is the slow one
    rate = b.whole_job_rate(32 * 100, w, ms)
    t0 = time.perf_counter()
    ref = b.run_reference(None, r, w) if r != 0 else "rank 0 runs the oracle"
    waited = time.perf_counter() - t0
    torch.distributed.barrier()
    torch.distributed.destroy_process_group()
    q.put((r, w, ms, rate, ref, waited))


def test_two_gloo_ranks_max_timing_and_reference_arm():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, w, ms, rate, ref, waited in res:
        assert w == 2 and ms == 15.0                           # every rank reports the slowest rank's time
        assert abs(rate - 2 * 3200 / 0.015) < 1e-6            # units of all ranks over that time
    assert res[1][4] is None and res[1][5] < 1.0               # the reference arm: rank 1 exits at once


def test_single_process_needs_no_process_group():
    b = _bench()
    assert b.max_over_ranks(7.5, 1, "cpu") == 7.5
    assert b.whole_job_rate(32, 1, 2.0) == 16000.0
