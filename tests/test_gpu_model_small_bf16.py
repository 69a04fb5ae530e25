"""Parity of the fused bf16 decode step on small shapes that the LLaMA
presets do not reach: head_dim 64, projections with fewer (block, k-block)
iterations than SMs (most CTAs idle in a projection), a batch above 16
(32-column accumulators), and run-to-run determinism of the decode step.

Accuracy bar: tests/_parity.storage_bar against the fp64 oracle (exact, and
with bf16 storage of the values the workload stores in bf16).
"""
import numpy as np
import pytest
import torch

import decoder_only_b200 as lb
import oracle
import synth
from synth.workloads import ModelShape, SEED
from _parity import greedy_bar, storage_bar

pytestmark = pytest.mark.gpu

# head_dim 64: 4 heads of 64; hidden 768; vocab 1024
SMALL64 = ModelShape("small-bf16-hd64", 2, 256, 4, 64, 768, 1024)
# head_dim 128: 4 heads of 128; hidden 1536; vocab 2048
SMALL128 = ModelShape("small-bf16-hd128", 2, 512, 4, 128, 1536, 2048)

PROMPT, STEPS = 40, 4


def _decode_vs_oracle(shape, B):
    toks = synth.tokens(SEED, B * (PROMPT + STEPS), shape.vocab).reshape(B, PROMPT + STEPS)
    m = lb.Model(shape, max_batch=B, max_seq=PROMPT + STEPS + 8)
    try:
        tk = torch.from_numpy(toks).cuda()
        pre = m.prefill(tk[:, :PROMPT].contiguous()).cpu().numpy()
        got = []
        for t in range(PROMPT, PROMPT + STEPS):
            _, lg = m.decode_step(tk[:, t].contiguous())
            got.append(lg.cpu().numpy())
        got = np.stack(got, axis=1)
    finally:
        m.close()
    exact, stored = oracle.prefill(shape, toks, storage=(None, "bf16"))
    storage_bar(pre, exact[:, :PROMPT], stored[:, :PROMPT], what=f"{shape.name} B={B} prefill")
    storage_bar(got, exact[:, PROMPT:], stored[:, PROMPT:], what=f"{shape.name} B={B} decode")
    greedy_bar(pre, exact[:, :PROMPT], stored[:, :PROMPT], what=f"{shape.name} B={B} prefill")
    greedy_bar(got, exact[:, PROMPT:], stored[:, PROMPT:], what=f"{shape.name} B={B} decode")


@pytest.mark.parametrize("shape,B", [(SMALL64, 3), (SMALL64, 20), (SMALL128, 1), (SMALL128, 32)])
def test_small_decode_against_oracle(shape, B):
    _decode_vs_oracle(shape, B)


@pytest.mark.parametrize("shape,B", [(SMALL128, 5), (SMALL64, 17)])
def test_decode_step_is_deterministic(shape, B):
    toks = synth.tokens(SEED + 1, B * (PROMPT + STEPS), shape.vocab).reshape(B, PROMPT + STEPS)
    m = lb.Model(shape, max_batch=B, max_seq=PROMPT + STEPS + 8)
    try:
        tk = torch.from_numpy(toks).cuda()
        m.prefill(tk[:, :PROMPT].contiguous(), logits=False)
        first = [m.decode_step(tk[:, t].contiguous())[1].clone() for t in range(PROMPT, PROMPT + STEPS)]
        m.rewind(PROMPT)
        again = [m.decode_step(tk[:, t].contiguous())[1].clone() for t in range(PROMPT, PROMPT + STEPS)]
    finally:
        m.close()
    for a, b in zip(first, again):
        assert torch.equal(a, b)
