"""The N > 1 path of bench.py on the CPU: two `gloo` ranks.

Decode and prefill shard as independent replicas (no collective on the data
path); the only cross-rank steps are the barrier around the timed region and
the max over ranks of its device time.  These tests run the host logic of
those steps with world_size 2."""
import io
import os
import contextlib
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench
from synth.workloads import LLAMA_7B, TINY


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = [12.5, 30.25][rank]
        dist.barrier()
        ms = bench.max_over_ranks(local_ms, world)
        value = bench.replica_throughput(world, 4 * 2048 + 4 * 128, 5, ms)
        toks = bench.replica_tokens(TINY, rank, 2, 16)
        # the reference arm: only rank 0 works and prints
        out = io.StringIO()
        if rank != 0:
            with contextlib.redirect_stdout(out):
                bench.run_reference(None, dict(batch=1, seq=8, decode=1, desc="x"), TINY)
        dist.barrier()
        q.put((rank, ms, value, toks.tolist(), out.getvalue()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_as_the_slowest_and_count_both_replicas():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, ms0, v0, t0, o0), (r1, ms1, v1, t1, o1) = res
    assert ms0 == ms1 == 30.25                       # every rank: the max over ranks
    assert v0 == v1 == pytest.approx(2 * (4 * 2048 + 4 * 128) * 5 / 30.25e-3)
    assert not np.array_equal(np.array(t0), np.array(t1))   # replicas draw their own prompts
    assert o1 == ""                                   # the reference arm prints on rank 0 only


def test_one_rank_needs_no_process_group():
    assert bench.max_over_ranks(7.0, 1) == 7.0
    assert bench.replica_throughput(1, 100, 2, 1000.0) == pytest.approx(200.0)
    assert bench.replica_tokens(LLAMA_7B, 0, 1, 4).shape == (1, 4)
