"""The host side of tensor-parallel prefill on the CPU: two `gloo` ranks.

Each rank builds the library's exchange callback (llama_allreduce_fn) the
way a GPU run does -- decoder_only_b200.allreduce_callback around
torch.distributed all-reduce (NCCL between GPUs, gloo here) -- and calls it
through its C function pointer on a host buffer, as the library calls it
between row blocks.  Checked: the blocks are summed over the ranks in place
and identically on both; a failing exchange reports non-zero; the ranks'
shard slices (llama_tp_shard) tile the heads and hidden units exactly.
"""
import ctypes
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from synth.workloads import LLAMA_7B, LLAMA_13B


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist

    import decoder_only_b200 as lb
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # a host "arena" standing in for the model's; trunk rows at an offset
        arena = torch.zeros(4096 + 64, dtype=torch.float32)
        rows = torch.arange(4096, dtype=torch.float32).reshape(64, 64)
        arena[64:] = (rows * (rank + 1) + 0.25 * rank).reshape(-1)
        base = arena.data_ptr()

        def resolve(ptr, count):
            off = (ptr - base) // 4
            return arena[off:off + count]

        cb = lb.allreduce_callback(resolve, lb.dist_allreduce())
        fn = ctypes.cast(cb, ctypes.c_void_p).value
        call = lb.ALLREDUCE_FN(fn)
        # three row blocks of the trunk, as the library exchanges them
        rcs = []
        for r0, nrows in ((0, 24), (24, 24), (48, 16)):
            rcs.append(call(base + 4 * (64 + r0 * 64), nrows * 64, None, None))
        # an exchange whose reduce raises reports failure instead of raising into C
        bad = lb.allreduce_callback(resolve, lambda buf, st: 1 / 0)
        rc_bad = bad(base, 8, None, None)
        # every rank's slices, gathered
        mine = [lb.tp_shard(s, rank, world) for s in (LLAMA_7B, LLAMA_13B, LLAMA_7B.with_(n_kv_heads=8))]
        allsh = [None] * world
        dist.all_gather_object(allsh, mine)
        q.put((rank, rcs, rc_bad, arena[64:].numpy().copy(), allsh))
    finally:
        dist.destroy_process_group()


def test_exchange_callback_sums_row_blocks_over_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        rank, rcs, rc_bad, buf, allsh = q.get(timeout=180)
        res[rank] = (rcs, rc_bad, buf, allsh)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    rows = np.arange(4096, dtype=np.float32)
    want = rows * 1 + rows * 2 + 0.25        # rank 0 + rank 1
    for rank in range(world):
        rcs, rc_bad, buf, allsh = res[rank]
        assert rcs == [0, 0, 0]
        assert rc_bad != 0
        assert np.array_equal(buf, want)
    assert np.array_equal(res[0][2], res[1][2])
    # the slices tile each model's heads, key/value heads and hidden units
    allsh = res[0][3]
    for i, shape in enumerate((LLAMA_7B, LLAMA_13B, LLAMA_7B.with_(n_kv_heads=8))):
        sl = [allsh[r][i] for r in range(world)]
        for key0, key, total in (("head0", "heads", shape.n_heads), ("kv_head0", "kv_heads", shape.kv_heads),
                                 ("hidden0", "hidden", shape.ffn_hidden)):
            covered = sorted(u for s in sl for u in range(s[key0], s[key0] + s[key]))
            assert covered == list(range(total))
