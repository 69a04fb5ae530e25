"""The paged KV cache ([NAR] "GQA Was Not an Original LLaMA Feature": decoding
keeps every earlier position's keys and values; here they live in pages of
128 positions from one pool, mapped per sequence by a page table).

A paged model and a contiguous one of the same shape and seed compute the
same thing on the same tokens: their logits must agree bit for bit, in
prefill and in decode steps that cross page boundaries, with a scrambled
page table (pages of one sequence scattered and out of order over the pool),
for ragged batches, grouped key/value heads and both head dims.  Checked
too: the table's validation and the positions it covers.
"""
import numpy as np
import pytest
import torch

import decoder_only_b200 as lb
import synth
from synth.workloads import LLAMA_7B, SEED, ModelShape

pytestmark = pytest.mark.gpu

SMALL128 = ModelShape("small-bf16-hd128", 2, 512, 4, 128, 1536, 2048)
SMALL64 = ModelShape("small-bf16-hd64", 2, 256, 4, 64, 768, 1024)
GQA2 = ModelShape("small-gqa2", 2, 512, 4, 128, 1536, 2048, n_kv_heads=2)
PAGE = 128


def _scrambled_table(B, pps, n_pages, seed):
    rng = np.random.default_rng(seed)
    pool = rng.permutation(n_pages)[: B * pps]
    return pool.reshape(B, pps).tolist()


def _run(m, toks, S, steps, lens=None):
    tk = torch.from_numpy(toks).cuda()
    pre = m.prefill(tk[:, :S].contiguous(), lens=lens).cpu().numpy()
    dec = []
    for t in range(S, S + steps):
        _, lg = m.decode_step(tk[:, t].contiguous())
        dec.append(lg.cpu().numpy())
    return pre, np.stack(dec, axis=1)


@pytest.mark.parametrize("shape,B,S,steps", [
    (SMALL128, 3, 254, 5),                 # decode crosses the page boundary at 256
    (SMALL64, 5, 300, 3),
    (GQA2, 4, 129, 2),
    (LLAMA_7B.with_(n_layers=2, name="llama-7b-2layer"), 2, 383, 3),
])
def test_paged_cache_equals_contiguous(shape, B, S, steps):
    max_seq = S + steps + 3
    pps = -(-max_seq // PAGE)
    n_pages = B * pps + 7
    toks = synth.tokens(SEED + 3, B * (S + steps), shape.vocab).reshape(B, S + steps)
    ref = lb.Model(shape, max_batch=B, max_seq=max_seq)
    try:
        want = _run(ref, toks, S, steps)
    finally:
        ref.close()
    m = lb.Model(shape, max_batch=B, max_seq=max_seq, kv_pages=n_pages)
    try:
        m.set_pages(_scrambled_table(B, pps, n_pages, 1))
        got = _run(m, toks, S, steps)
    finally:
        m.close()
    for a, b in zip(got, want):
        assert np.array_equal(a, b)


def test_paged_ragged_batch_equals_contiguous():
    shape, B, S, steps = SMALL128, 3, 260, 4
    lens = [260, 100, 131]
    max_seq = S + steps
    pps = -(-max_seq // PAGE)
    toks = synth.tokens(SEED + 4, B * (S + steps), shape.vocab).reshape(B, S + steps)
    ref = lb.Model(shape, max_batch=B, max_seq=max_seq)
    try:
        tk = torch.from_numpy(toks).cuda()
        ref.prefill(tk[:, :S].contiguous(), lens=lens, logits=False)
        want = [ref.decode_step(tk[:, S + i].contiguous())[1].cpu().numpy() for i in range(steps)]
    finally:
        ref.close()
    m = lb.Model(shape, max_batch=B, max_seq=max_seq, kv_pages=B * pps)
    try:
        m.set_pages(_scrambled_table(B, pps, B * pps, 2))
        m.prefill(tk[:, :S].contiguous(), lens=lens, logits=False)
        got = [m.decode_step(tk[:, S + i].contiguous())[1].cpu().numpy() for i in range(steps)]
    finally:
        m.close()
    for a, b in zip(got, want):
        assert np.array_equal(a, b)


def test_page_table_validation_and_coverage():
    shape = SMALL64
    m = lb.Model(shape, max_batch=2, max_seq=512, kv_pages=5)    # fewer than 2 x 4 pages: no default table
    try:
        tok = torch.zeros(2, 200, dtype=torch.int32, device="cuda")
        with pytest.raises(lb.LlamaError) as e:
            m.prefill(tok, logits=False)
        assert e.value.code == -5                                  # no table yet
        for bad in ([[0, 1], [1, 2]], [[0, 5], [1, 2]], [[0, -1], [2, 3]]):   # repeated, out of range
            with pytest.raises(lb.LlamaError) as e:
                m.set_pages(bad)
            assert e.value.code == -1
        m.set_pages([[4, 0], [2, 3]])                              # 2 pages each: 256 positions
        m.prefill(tok, logits=False)
        with pytest.raises(lb.LlamaError) as e:
            m.prefill(torch.zeros(2, 257, dtype=torch.int32, device="cuda"), logits=False)
        assert e.value.code == -1                                  # beyond the sequences' pages
        m.prefill(torch.zeros(2, 255, dtype=torch.int32, device="cuda"), logits=False)
        m.decode_step(torch.zeros(2, dtype=torch.int32, device="cuda"))   # position 255: the last covered
        with pytest.raises(lb.LlamaError) as e:
            m.decode_step(torch.zeros(2, dtype=torch.int32, device="cuda"))
        assert e.value.code == -5
    finally:
        m.close()
