"""The 33B shape (d 6656 = 52 heads of 128, hidden 17920, vocab 32000):
two layers at these widths against the fp64 oracle, prefill and greedy
decode, under the derived bf16 storage bar (tests/_parity.storage_bar).
52 heads and 52 / 140 row blocks of 128 in the d- and h-wide projections:
the projection tilings, the stream-K ranges and the attention split meet
counts the 7B and 13B presets do not."""
import numpy as np
import pytest
import torch

import decoder_only_b200 as lb
import oracle
import synth
from synth.workloads import LLAMA_33B, SEED
from _parity import greedy_bar, storage_bar

pytestmark = pytest.mark.gpu

SHAPE = LLAMA_33B.with_(n_layers=2, name="llama-33b-2layer")
B, PROMPT, STEPS = 2, 64, 3


def test_33b_widths_prefill_and_decode_against_oracle():
    toks = synth.tokens(SEED, B * (PROMPT + STEPS), SHAPE.vocab).reshape(B, PROMPT + STEPS)
    m = lb.Model(SHAPE, max_batch=B, max_seq=PROMPT + STEPS + 16)
    try:
        tk = torch.from_numpy(toks).cuda()
        pre = m.prefill(tk[:, :PROMPT].contiguous()).cpu().numpy()
        dec = []
        for t in range(PROMPT, PROMPT + STEPS):
            _, lg = m.decode_step(tk[:, t].contiguous())
            dec.append(lg.cpu().numpy())
        dec = np.stack(dec, axis=1)
    finally:
        m.close()
        torch.cuda.empty_cache()
    exact, stored = oracle.prefill(SHAPE, toks, storage=(None, "bf16"))
    storage_bar(pre, exact[:, :PROMPT], stored[:, :PROMPT], what="33B prefill")
    storage_bar(dec, exact[:, PROMPT:], stored[:, PROMPT:], what="33B decode")
    greedy_bar(pre, exact[:, :PROMPT], stored[:, :PROMPT], what="33B prefill")
    greedy_bar(dec, exact[:, PROMPT:], stored[:, PROMPT:], what="33B decode")
