"""Tensor-parallel prefill ([KN] "Efficient Training Implementation": the
model split across GPUs, the all-reduce hidden behind computation), parity
against the oracle.

The shards run on one GPU, each in its own host thread and stream, with the
exchange of tests/_tp.LocalGroup in place of NCCL (every run here has one
GPU): the library's side -- sliced weights, partial O and down products,
the row-block schedule on two streams -- is the one a multi-GPU run uses.
Checked: every shard ends with the same logits (bit for bit); the logits
match the fp64 oracle of the unsharded model under the bars of
tests/_parity.py (fp32: 1e-4 RMS); the row-block count does not change a
bit of the result; decoding on a shard is refused.
"""
import numpy as np
import pytest
import torch

import decoder_only_b200 as lb
import oracle
import synth
from synth.workloads import BLOCK_7B, LLAMA_7B, SEED, TINY, ModelShape
from _parity import greedy_bar, rms, storage_bar
from _tp import run_shards

pytestmark = pytest.mark.gpu


def _prefill_all(tokens):
    def work(m, r):
        return m.prefill(torch.from_numpy(tokens).cuda()).cpu().numpy()
    return work


def _same_on_every_shard(outs):
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])
    return outs[0]


def test_two_shards_7b_widths_against_oracle():
    shape = LLAMA_7B.with_(n_layers=2, name="llama-7b-2layer")
    B, S = 2, 384
    toks = synth.tokens(SEED + 7, B * S, shape.vocab).reshape(B, S)
    got = _same_on_every_shard(run_shards(shape, 2, B, S, _prefill_all(toks), chunks=3))
    exact, stored = oracle.prefill(shape, toks, storage=(None, "bf16"))
    storage_bar(got, exact, stored, what="TP=2 7B widths")
    greedy_bar(got, exact, stored, what="TP=2 7B widths")


def test_row_blocks_do_not_change_the_result():
    shape = LLAMA_7B.with_(n_layers=1, name="llama-7b-1layer")
    B, S = 3, 200                         # 600 rows: blocks of 128 / 256 / 640 rows, ragged last block
    toks = synth.tokens(SEED + 8, B * S, shape.vocab).reshape(B, S)
    ref = run_shards(shape, 2, B, S, _prefill_all(toks), chunks=1)
    for chunks in (2, 5):
        got = run_shards(shape, 2, B, S, _prefill_all(toks), chunks=chunks)
        for a, b in zip(got, ref):
            assert np.array_equal(a, b)


def test_one_7b_block_on_the_trunk_two_shards():
    B, S = 1, 2048
    x = synth.normal_f32(SEED, synth.TRUNK, S * BLOCK_7B.d_model, 1.0).reshape(S, BLOCK_7B.d_model)

    def work(m, r):
        return m.prefill_trunk(torch.from_numpy(x).cuda()[None]).cpu().numpy()[0].astype(np.float64)

    y = _same_on_every_shard(run_shards(BLOCK_7B, 2, B, S, work))
    x64 = x.astype(np.float64)
    W = oracle.layer_weights(BLOCK_7B, 0)
    ref = oracle.block_forward(BLOCK_7B, x64, weights=W)
    ref16 = oracle.block_forward(BLOCK_7B, x64, weights=W, storage="bf16")
    storage_bar(y, ref, ref16, what="TP=2 7B block y")
    storage_bar(y - x64, ref - x64, ref16 - x64, what="TP=2 7B block y - x")


@pytest.mark.parametrize("shape,T", [
    (ModelShape("tp-hd128", 2, 512, 4, 128, 1536, 2048), 4),
    (ModelShape("tp-gqa2", 2, 512, 4, 128, 1536, 2048, n_kv_heads=2), 2),
    (ModelShape("tp-bias-hd64", 2, 256, 4, 64, 768, 1024, bias=True), 2),
])
def test_small_shapes_against_oracle(shape, T):
    B, S = 3, 96
    toks = synth.tokens(SEED + 9, B * S, shape.vocab).reshape(B, S)
    got = _same_on_every_shard(run_shards(shape, T, B, S, _prefill_all(toks)))
    exact, stored = oracle.prefill(shape, toks, storage=(None, "bf16"))
    storage_bar(got, exact, stored, what=f"TP={T} {shape.name}")
    greedy_bar(got, exact, stored, what=f"TP={T} {shape.name}")


def test_fp32_tiny_two_shards_within_1e4():
    B, S = 2, 32
    toks = synth.tokens(SEED, B * S, TINY.vocab).reshape(B, S)
    got = _same_on_every_shard(run_shards(TINY, 2, B, S, _prefill_all(toks), chunks=2))
    exact = oracle.prefill(TINY, toks)
    err = float(np.max(np.abs(got - exact)))
    print("TP=2 tiny fp32 max|err|/RMS:", err / rms(exact))
    assert err <= 1e-4 * rms(exact)
    greedy_bar(got, exact, what="TP=2 tiny fp32")


def test_a_shard_refuses_decoding_and_needs_its_exchange():
    shape = ModelShape("tp-small", 1, 256, 4, 64, 768, 1024)
    m = lb.Model(shape, max_batch=2, max_seq=16, tp=(1, 2))
    try:
        tok = torch.zeros(2, 8, dtype=torch.int32, device="cuda")
        with pytest.raises(lb.LlamaError) as e:
            m.prefill(tok)
        assert e.value.code == -5                     # no exchange installed
        with pytest.raises(lb.LlamaError) as e:
            m.decode_step(tok[:, 0].contiguous())
        assert e.value.code == -1
    finally:
        m.close()
