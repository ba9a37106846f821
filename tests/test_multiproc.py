"""The replica (multi-GPU) host logic of bench.py, as two gloo ranks on the CPU.

The block does not shard: N GPUs run N independent replicas.  What needs
checking without GPUs is the host plumbing: every rank takes part in the same
max-reduction of its timing, the job value counts all ranks' tokens over the
slowest rank's time, and ranks process different token batches.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    from moe_inputs import CONFIGS
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        my_ms = 10.0 + 5.0 * rank
        ms = bench.max_over_ranks(my_ms, world, torch.device("cpu"))
        value = bench.job_tokens_per_s(ms, 32, 4, world)
        x = bench.replica_tokens(CONFIGS["tiny"], rank)
        q.put((rank, ms, value, x[0, :8].tolist()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_replicas_agree_on_max_time_and_job_value():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    ms = [r[1] for r in res]
    assert ms == [15.0, 15.0]                     # max over ranks, seen by every rank
    expected = world * 32 * 4 / (15.0 / 1e3)
    assert all(abs(r[2] - expected) < 1e-6 * expected for r in res)
    assert res[0][3] != res[1][3]                 # independent token batches
