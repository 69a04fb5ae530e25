"""Grouped keys and values (GQA / MQA, the pages' next step for decode
bandwidth: [NAR] "GQA Was Not an Original LLaMA Feature"): n_kv key/value
heads, query head h reading key/value head h / (H / n_kv).  Prefill and
greedy decode against the fp64 oracle with the same grouping, under the
derived bf16 storage bar (tests/_parity.storage_bar) or the fp32 1e-4 bound.
"""
import numpy as np
import pytest
import torch

import decoder_only_b200 as lb
import oracle
import synth
from synth.workloads import LLAMA_7B, ModelShape, SEED, TINY
from _parity import greedy_bar, rms, storage_bar

pytestmark = pytest.mark.gpu

PROMPT, STEPS = 40, 3


def _run(shape, B, prompt=PROMPT, steps=STEPS):
    toks = synth.tokens(SEED + 5, B * (prompt + steps), shape.vocab).reshape(B, prompt + steps)
    m = lb.Model(shape, max_batch=B, max_seq=prompt + steps + 8)
    try:
        tk = torch.from_numpy(toks).cuda()
        pre = m.prefill(tk[:, :prompt].contiguous()).cpu().numpy()
        dec = []
        for t in range(prompt, prompt + steps):
            _, lg = m.decode_step(tk[:, t].contiguous())
            dec.append(lg.cpu().numpy())
    finally:
        m.close()
        torch.cuda.empty_cache()
    got = np.concatenate([pre, np.stack(dec, axis=1)], axis=1)
    return got, toks


@pytest.mark.parametrize("shape,B", [
    (ModelShape("mqa-hd128", 2, 512, 4, 128, 1536, 2048, n_kv_heads=1), 3),
    (ModelShape("gqa2-hd128", 2, 512, 4, 128, 1536, 2048, n_kv_heads=2), 5),
    (ModelShape("gqa4-hd64", 2, 512, 8, 64, 1536, 2048, n_kv_heads=2), 2),
    (ModelShape("gqa2-hd64", 2, 256, 4, 64, 768, 1024, n_kv_heads=2), 17),
])
def test_grouped_kv_prefill_and_decode_against_oracle(shape, B):
    got, toks = _run(shape, B)
    exact, stored = oracle.prefill(shape, toks, storage=(None, "bf16"))
    storage_bar(got, exact, stored)
    greedy_bar(got, exact, stored)


def test_grouped_kv_fp32_model_within_1e4():
    shape = TINY.with_(n_kv_heads=2, name="tiny-gqa2")
    got, toks = _run(shape, 2, prompt=24)
    exact = oracle.prefill(shape, toks)
    err = np.max(np.abs(got - exact))
    assert err <= 1e-4 * rms(exact), (err, rms(exact))


def test_grouped_kv_7b_widths_two_layers():
    """d 4096, 32 query heads sharing 8 key/value heads (groups of 4)."""
    shape = LLAMA_7B.with_(n_layers=2, n_kv_heads=8, name="llama-7b-gqa8-2layer")
    got, toks = _run(shape, 2, prompt=48, steps=2)
    exact, stored = oracle.prefill(shape, toks, storage=(None, "bf16"))
    storage_bar(got, exact, stored)
    greedy_bar(got, exact, stored)


def test_grouped_kv_cache_is_n_kv_heads_wide():
    shape = ModelShape("gqa2-hd128", 1, 512, 4, 128, 1536, 2048, n_kv_heads=2)
    m = lb.Model(shape, max_batch=2, max_seq=32)
    try:
        kv = m.tensor("kv")
        # [L][2][max_batch][n_kv][max_seq][hd]
        assert kv.numel() == 1 * 2 * 2 * 2 * 32 * 128 * 2      # bf16 bytes
    finally:
        m.close()


def test_grouped_kv_shapes_are_validated():
    with pytest.raises(lb.LlamaError):
        lb.Model(ModelShape("bad", 1, 512, 4, 128, 1536, 2048, n_kv_heads=3), max_batch=1, max_seq=8)
