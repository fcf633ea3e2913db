"""Multi-rank host logic of bench.py on CPU: world size 2 over gloo.

The path shards by (batch, head) with no data-path collective; the only
collectives are the timing barrier and the max-over-ranks reduction.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ms_local = 10.0 + 5.0 * rank                     # rank 1 is the slow one
        dist.barrier()
        ms = bench.max_over_ranks(ms_local, world)
        value = bench.job_throughput(16384, world, 100, ms)
        # each rank draws its own batch (seed = rank): different data, same shapes
        from chunked_gated_delta_14_b200.inputs import make_inputs, workload
        x = make_inputs(workload("gdn_bf16", B=1, H=1, T=64), seed=rank)
        q.put((rank, ms, value, float(x["q"].float().sum())))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_world2():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, ms, value, _ in got:
        assert ms == 15.0                                # the slowest rank's time, on every rank
        assert value == pytest.approx(16384 * 2 * 100 / 0.015)
    assert got[0][3] != got[1][3]                        # independent batches per rank


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_throughput(10, 1, 4, 2.0) == pytest.approx(10 * 4 / 0.002)


def test_reference_arm_other_ranks_do_no_work():
    import argparse
    import bench
    args = argparse.Namespace(steps=1, warmup=3, ref_budget=1.0, batch=0)
    # rank 1 of 2 returns at once: no oracle import, no output
    assert bench.run_reference(args, rank=1, world=2) is None
