"""Ragged batches: sequences of different prompt lengths in one [B, S] block
(llama_prefill_ragged), then greedy decode steps in which every sequence
continues at its own position.  Each sequence is checked against the fp64
oracle run on that sequence alone: prefill rows 0..len-1 and the decode
steps (teacher-forced), under the derived bf16 storage bar
(tests/_parity.storage_bar) or, for the fp32 model, the 1e-4 RMS bound.
Padding tokens after a sequence's length are arbitrary valid ids."""
import numpy as np
import pytest
import torch

import decoder_only_b200 as lb
import oracle
import synth
from synth.workloads import ModelShape, SEED, TINY
from _parity import greedy_bar, rms, storage_bar

pytestmark = pytest.mark.gpu

SMALL64 = ModelShape("small-bf16-hd64", 2, 256, 4, 64, 768, 1024)
SMALL128 = ModelShape("small-bf16-hd128", 2, 512, 4, 128, 1536, 2048)
STEPS = 3


def _run(shape, lens, seed):
    B, S = len(lens), max(lens)
    toks = synth.tokens(SEED + seed, B * (S + STEPS), shape.vocab).reshape(B, S + STEPS)
    m = lb.Model(shape, max_batch=B, max_seq=S + STEPS + 8)
    try:
        pre = m.prefill(torch.from_numpy(toks[:, :S].copy()).cuda(), lens=lens).cpu().numpy()
        assert m.positions() == list(lens)
        assert m.position == S
        dec = []
        for i in range(STEPS):
            step = torch.tensor([toks[b, lens[b] + i] for b in range(B)], dtype=torch.int32).cuda()
            _, lg = m.decode_step(step)
            dec.append(lg.cpu().numpy())
        assert m.positions() == [n + STEPS for n in lens]
    finally:
        m.close()
    dec = np.stack(dec, axis=1)            # [B, STEPS, V]
    got, ex, st = [], [], []
    for b in range(B):
        n = lens[b]
        e, s = oracle.prefill(shape, toks[b:b + 1, :n + STEPS], storage=(None, "bf16"))
        got.append(np.concatenate([pre[b, :n], dec[b]]))
        ex.append(e[0])
        st.append(s[0])
    return np.concatenate(got), np.concatenate(ex), np.concatenate(st)


@pytest.mark.parametrize("shape,lens", [
    (SMALL128, [40, 7, 33, 1, 25]),
    (SMALL64, [12, 48, 3, 30, 48, 17, 1, 9, 40, 22, 5, 48, 36, 2, 28, 44, 19]),   # 17 sequences: 32-column tiles
    (SMALL128, [64, 2]),
])
def test_ragged_prefill_and_decode_against_oracle(shape, lens):
    got, exact, stored = _run(shape, lens, 11)
    storage_bar(got, exact, stored)
    greedy_bar(got, exact, stored)


def test_ragged_fp32_model_within_1e4():
    lens = [29, 4, 17]
    got, exact, _ = _run(TINY, lens, 12)
    err = np.max(np.abs(got - exact))
    assert err <= 1e-4 * rms(exact), (err, rms(exact))


def test_ragged_greedy_continues_from_each_last_prompt_row():
    lens = [21, 6, 14, 30]
    B, S = len(lens), max(lens)
    toks = synth.tokens(SEED + 13, B * S, SMALL128.vocab).reshape(B, S)
    m = lb.Model(SMALL128, max_batch=B, max_seq=S + 8)
    try:
        tk = torch.from_numpy(toks).cuda()
        lg = m.prefill(tk, lens=lens)
        choice = torch.stack([lg[b, lens[b] - 1].argmax() for b in range(B)]).to(torch.int32)
        # generate's first step consumes the prefill's greedy choice at row lens[b] - 1 ...
        gen = m.generate(None, 2, batch=B)
        assert m.positions() == [n + 2 for n in lens]
        # ... exactly as a decode step fed that choice explicitly
        m.prefill(tk, lens=lens)
        nxt, _ = m.decode_step(choice, logits=False)
        assert torch.equal(gen[0], nxt)
        with pytest.raises(lb.LlamaError):
            m.rewind(min(lens) + 3)     # beyond the shortest sequence's cache
        m.rewind(min(lens))
        assert m.positions() == [min(lens)] * B
    finally:
        m.close()


def test_ragged_lengths_are_validated():
    m = lb.Model(SMALL128, max_batch=2, max_seq=16)
    try:
        t = torch.zeros(2, 8, dtype=torch.int32, device="cuda")
        for bad in ([0, 4], [9, 4], [3, -1]):
            with pytest.raises(lb.LlamaError):
                m.prefill(t, lens=bad)
    finally:
        m.close()
