"""Parity of the bf16 7B-shaped paths at their full sizes.

Accuracy bars (tests/_parity.py): the GPU must be no further from the exact
fp64 oracle than bf16 storage of the values the workload stores in bf16
moves the oracle itself (x1.25 RMS, x1.5 max), and may change no more greedy
tokens than that storage does.  The stated 2e-2 max-norm figure is printed
for every comparison; bf16 storage alone exceeds it at one block
(tests/test_oracle_pins.py::test_bf16_storage_alone_moves_one_7b_block_past_2e2)
and at depth (test_bf16_kv_cache_alone_moves_deep_logits_past_2e2).

 * one 7B block on an N(0,1) fp32 trunk, 1 x 2048 (y and the block's
   increment y - x);
 * the 32-layer model, prefill 4 x 2048: sampled rows (whole rows of two
   sequences, positions 0..99) against the oracle -- exact by causality;
 * greedy decode against the oracle (prompt 96, teacher-forced steps 96..99);
 * decode at the full cache length (positions 2048..2051) against prefill
   rows of the extended sequences, and the invariants (causality, prefix
   truncation, run-to-run determinism) at full size.
"""
import numpy as np
import pytest
import torch

import decoder_only_b200 as lb
import oracle
import synth
from synth.workloads import BLOCK_7B, LLAMA_7B, SEED
from _parity import argmax_agreement, greedy_bar, rms, storage_bar

pytestmark = pytest.mark.gpu
B, S, STEPS = 4, 2048, 128


def test_single_block_7b():
    m = lb.Model(BLOCK_7B, max_batch=1, max_seq=S)
    try:
        x = synth.normal_f32(SEED, synth.TRUNK, S * BLOCK_7B.d_model, 1.0).reshape(S, BLOCK_7B.d_model)
        y = m.prefill_trunk(torch.from_numpy(x).cuda()[None]).cpu().numpy()[0].astype(np.float64)
    finally:
        m.close()
    x64 = x.astype(np.float64)
    W = oracle.layer_weights(BLOCK_7B, 0)
    ref = oracle.block_forward(BLOCK_7B, x64, weights=W)
    ref16 = oracle.block_forward(BLOCK_7B, x64, weights=W, storage="bf16")
    storage_bar(y, ref, ref16, what="7B block y")
    storage_bar(y - x64, ref - x64, ref16 - x64, what="7B block y - x")
    # largest feature of each row's increment: the block's own "greedy" choice
    greedy_bar(y - x64, ref - x64, ref16 - x64, what="7B block, argmax of y - x per row")


@pytest.fixture(scope="module")
def model():
    m = lb.Model(LLAMA_7B, max_batch=B, max_seq=S + STEPS)
    yield m
    m.close()
    torch.cuda.empty_cache()


@pytest.fixture(scope="module")
def tokens():
    return synth.tokens(SEED, B * (S + STEPS), LLAMA_7B.vocab).reshape(B, S + STEPS)


@pytest.fixture(scope="module")
def oracle_rows(tokens):
    """Oracle logits of sequences 0 and 3, positions 0..99: exact, and with
    bf16 storage of the values the workload stores in bf16."""
    exact, stored = oracle.prefill(LLAMA_7B, tokens[[0, 3], :100], storage=(None, "bf16"))
    return exact, stored


def test_prefill_full_size_sampled_rows(model, tokens, oracle_rows):
    lg = model.prefill(torch.from_numpy(tokens[:, :S].copy()).cuda())
    got = lg[[0, 3], :100].cpu().numpy()
    exact, stored = oracle_rows
    storage_bar(got, exact, stored, what="7B prefill rows")
    greedy_bar(got, exact, stored, what="7B prefill rows")
    # every row is finite and on the oracle's scale
    r = lg.float()
    assert torch.isfinite(r).all()
    assert abs(float(r.std()) / rms(exact) - 1.0) < 0.1


def test_greedy_decode_against_oracle(model, tokens, oracle_rows):
    model.prefill(torch.from_numpy(tokens[:, :96].copy()).cuda(), logits=False)
    got = []
    for t in range(96, 100):
        _, lg = model.decode_step(torch.from_numpy(tokens[:, t].copy()).cuda())
        got.append(lg[[0, 3]].cpu().numpy())
    got = np.stack(got, axis=1)
    exact, stored = oracle_rows
    storage_bar(got, exact[:, 96:100], stored[:, 96:100], what="7B decode 96..99")
    greedy_bar(got, exact[:, 96:100], stored[:, 96:100], what="7B decode 96..99")


def test_full_length_decode_equals_prefill_rows(model, tokens, oracle_rows):
    tk = torch.from_numpy(tokens).cuda()
    model.prefill(tk[:, :S].contiguous(), logits=False)
    dec = []
    for t in range(S, S + 4):
        _, lg = model.decode_step(tk[:, t].contiguous())
        dec.append(lg.cpu().numpy())
    dec = np.stack(dec, axis=1)
    ref = model.prefill(tk[:, :S + 4].contiguous())[:, S:S + 4].cpu().numpy()
    # two bf16 computations of the same rows (split-K decode GEMMs and decode
    # attention vs prefill kernels): each within the storage bar of the exact
    # answer, so their difference within twice it
    exact, stored = oracle_rows
    r = rms(exact)
    bar_rms = rms(stored - exact) / r
    bar_max = float(np.max(np.abs(stored - exact))) / r
    diff = dec - ref
    print("decode vs prefill:", rms(diff) / rms(ref), np.max(np.abs(diff)) / rms(ref), bar_rms, bar_max)
    assert rms(diff) / rms(ref) <= 2 * 1.5 * bar_rms
    assert np.max(np.abs(diff)) / rms(ref) <= 2 * 2.0 * bar_max
    # consistency of two GPU paths, not parity (the oracle comparison at this
    # cache length is tests/test_gpu_decode_long_cache.py): printed only
    print("decode vs prefill greedy agreement (strict, near-tie):", argmax_agreement(dec, ref))


def test_generate_full_length_is_greedy(model, tokens):
    tk = torch.from_numpy(tokens).cuda()
    model.prefill(tk[:, :S].contiguous(), logits=False)
    out = model.generate(tk[:, S].contiguous(), 8).cpu().numpy()
    assert out.shape == (8, B) and out.min() >= 0 and out.max() < LLAMA_7B.vocab
    assert model.position == S + 8


def test_causality_prefix_and_determinism_full_size(model, tokens):
    tk = torch.from_numpy(tokens[:, :S].copy()).cuda()
    a = model.prefill(tk)
    b = model.prefill(tk)
    assert torch.equal(a, b)                                   # run to run
    t2 = tk.clone()
    t2[:, 1000:] = (t2[:, 1000:] + 7) % LLAMA_7B.vocab
    c = model.prefill(t2)
    assert torch.equal(c[:, :1000], a[:, :1000])               # causality
    assert not torch.equal(c[:, 1000:], a[:, 1000:])
    d = model.prefill(tk[:, :640].contiguous())
    assert torch.allclose(d, a[:, :640], rtol=0, atol=1e-5 * float(a.std()))   # prefix truncation
