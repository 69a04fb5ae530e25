"""The fused decode step at the full cache length, against the oracle.

A two-layer model at 7B widths (d 4096, 32 heads of 128, hidden 11008, vocab
32000) takes the bench's batch and prompt length, 4 prompts of 2048 tokens,
and then three teacher-forced decode steps at positions 2048, 2049 and 2050
([NAR] "GQA Was Not an Original LLaMA Feature": each step reads the keys
and values of every earlier position).  At this length the decode step's
attention cuts each (sequence, head) pair's 129 sixteen-key chunks across
several ranges of attention warps and merges the ranges' partial softmax
results: the regime the bench times.  Sequences 0 and 3 are compared with the
fp64 oracle run on each sequence alone (sequences are independent), under
the bars of tests/_parity.py.
"""
import numpy as np
import pytest
import torch

import decoder_only_b200 as lb
import oracle
import synth
from synth.workloads import LLAMA_7B, SEED
from _parity import greedy_bar, storage_bar

pytestmark = pytest.mark.gpu

SHAPE = LLAMA_7B.with_(n_layers=2, name="llama-7b-2layer")
B, S, STEPS = 4, 2048, 3
CHECKED = [0, 3]


def test_decode_at_positions_2048_to_2050_against_oracle():
    toks = synth.tokens(SEED + 5, B * (S + STEPS), SHAPE.vocab).reshape(B, S + STEPS)
    m = lb.Model(SHAPE, max_batch=B, max_seq=S + 16)
    try:
        tk = torch.from_numpy(toks).cuda()
        m.prefill(tk[:, :S].contiguous(), logits=False)
        got = []
        for t in range(S, S + STEPS):
            _, lg = m.decode_step(tk[:, t].contiguous())     # teacher-forced: the prompt's next token
            got.append(lg[CHECKED].cpu().numpy())
        assert m.position == S + STEPS
    finally:
        m.close()
        torch.cuda.empty_cache()
    got = np.stack(got, axis=1)                              # (2, STEPS, V)
    exact, stored = oracle.prefill(SHAPE, toks[CHECKED], storage=(None, "bf16"))
    exact, stored = exact[:, S:], stored[:, S:]
    storage_bar(got, exact, stored, what="decode at positions 2048..2050")
    greedy_bar(got, exact, stored, what="decode at positions 2048..2050")
