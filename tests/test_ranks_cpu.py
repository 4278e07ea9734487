"""The multi-process path of bench.py on CPU: two gloo ranks on 127.0.0.1.

Each rank runs its own batch (weak scaling, no data-path collective); the
only collectives are the barrier and the max-over-ranks reduction of the
step time, and the job's value is every rank's flops over the slowest
rank's time.  These are checked here with real processes; the GPU work of a
rank is the single-GPU path covered by the gpu tests."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        ms = bench.max_over_ranks(2.0 + 3.0 * rank, "cpu")   # rank r took 2 + 3r ms
        value = bench.job_value(5e12, ms, world)
        dist.barrier()
        q.put((rank, ms, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_to_the_slowest():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, value in got:
        assert ms == 5.0                                   # the slowest rank's time, on every rank
        assert value == pytest.approx(2 * 5e12 / 5e-3 / 1e12)  # both ranks' flops over it


def test_single_process_needs_no_group():
    import bench
    assert bench.max_over_ranks(3.5, "cpu") == 3.5
    assert bench.job_value(1e12, 1.0, 1) == pytest.approx(1000.0)


def test_ranks_draw_independent_batches():
    from workloads import WORKLOADS, make_qkv
    w = WORKLOADS["tiny"]
    q0, _, _ = make_qkv(w, seed=0)
    q1, _, _ = make_qkv(w, seed=1)
    q0b, _, _ = make_qkv(w, seed=0)
    assert np.array_equal(q0, q0b) and not np.array_equal(q0, q1)
