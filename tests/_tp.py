"""Tensor-parallel shards of one model on one GPU, for the parity tests.

Each shard is driven by its own host thread on its own CUDA stream, exactly
as the shards of a multi-GPU run are driven by their own processes; only the
exchange differs.  LocalGroup's exchange sums the shards' buffers in rank
order on each shard's stream (so every shard gets the same bits, as NCCL
gives every rank), ordered by CUDA events: a shard reads the others'
buffers only after their producers, and overwrites its own only after
every shard has read it.  No kernel waits on another: the order is carried
by stream dependencies on work already queued.
"""
import threading

import torch

import decoder_only_b200 as lb


class LocalGroup:
    def __init__(self, size: int):
        self.size = size
        self.bar = threading.Barrier(size, timeout=300)   # a shard that never arrives fails the test
        self.bufs = [None] * size
        self.ready = [None] * size
        self.read = [None] * size

    def reduce_for(self, rank: int):
        def reduce(buf, stream):
            ev = torch.cuda.Event()
            ev.record(stream)
            self.bufs[rank], self.ready[rank] = buf, ev
            self.bar.wait()                               # every shard's block and its producer event
            for k in range(self.size):
                if k != rank:
                    stream.wait_event(self.ready[k])
            with torch.cuda.stream(stream):
                total = self.bufs[0].clone()
                for k in range(1, self.size):
                    total.add_(self.bufs[k])
            done = torch.cuda.Event()
            done.record(stream)
            self.read[rank] = done
            self.bar.wait()                               # every shard has queued its reads
            for k in range(self.size):
                if k != rank:
                    stream.wait_event(self.read[k])
            with torch.cuda.stream(stream):
                buf.copy_(total)
        return reduce


def run_shards(shape, size: int, max_batch: int, max_seq: int, work, chunks: int = 4):
    """Builds `size` shards of `shape`, installs a LocalGroup exchange, and
    runs work(model, rank) on every shard at once, each in its own thread and
    stream.  Returns the list of results (rank order)."""
    models = [lb.Model(shape, max_batch=max_batch, max_seq=max_seq, tp=(r, size)) for r in range(size)]
    group = LocalGroup(size)
    for r, m in enumerate(models):
        m.set_allreduce(group.reduce_for(r), chunks=chunks)
    out = [None] * size
    errs = []

    def body(r):
        try:
            torch.cuda.set_device(0)
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                out[r] = work(models[r], r)
            s.synchronize()
        except BaseException as e:   # reported by the caller
            errs.append(e)
            group.bar.abort()

    threads = [threading.Thread(target=body, args=(r,)) for r in range(size)]
    try:
        for t in threads:
            t.start()
        for t in threads:
            t.join()
    finally:
        for m in models:
            m.close()
    if errs:
        raise errs[0]
    return out
