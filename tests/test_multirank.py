"""Multi-rank logic of bench.py on CPU with gloo, world size 2: the max over
ranks of the device time, the barrier, the whole-job (weak scaling) value,
and the reference arm running on rank 0 only."""
import multiprocessing as mp
import os
import socket

import pytest


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, init_method=f"tcp://127.0.0.1:{port}")
    try:
        ms_local = [2.0, 3.5][rank]  # rank 1 is the slow one
        ms = bench.reduce_max(ms_local, world)
        bench.barrier(world)
        value = bench.weak_scaling_value(1e12, world, ms)
        args = bench.parse_args(["--impl", "reference", "--steps", "1", "--warmup", "3"])
        ref = bench.run_reference(args, rank, world) if rank != 0 else "rank0-skipped"
        q.put((rank, ms, value, ref))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_is_max_over_ranks_and_value_is_whole_job():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(2):
        rank, ms, value, ref = q.get(timeout=120)
        out[rank] = (ms, value, ref)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out[0][0] == out[1][0] == 3.5
    # two ranks x 1e12 FLOPs in 3.5 ms = 571.4 TFLOP/s for the whole job
    assert abs(out[0][1] - 2e12 / 3.5e-3 / 1e12) < 1e-9
    assert out[1][2] is None  # the reference arm does no work off rank 0


def test_single_rank_helpers_are_identities():
    import bench
    assert bench.reduce_max(1.25, 1) == 1.25
    bench.barrier(1)
    assert abs(bench.weak_scaling_value(2e12, 1, 2.0) - 1000.0) < 1e-9
