"""End-to-end parity of the fp32 tiny LLaMA (2 layers, d=128, 4 heads x 32,
hidden 512, vocab 1000): prefill logits and greedy decode against the fp64
oracle at max|err| <= 1e-4 RMS(ref)."""
import numpy as np
import pytest
import torch

import decoder_only_b200 as lb
import oracle
import synth
from synth.workloads import TINY
from _parity import rel_max_err, argmax_agreement, greedy_bar

pytestmark = pytest.mark.gpu
TOL = 1e-4


@pytest.fixture(scope="module")
def model():
    m = lb.Model(TINY, max_batch=3, max_seq=64)
    yield m
    m.close()


def _tok(B, S, first=0):
    return synth.tokens(synth.workloads.SEED, B * S, TINY.vocab, first=first).reshape(B, S)


def test_weights_on_device_equal_the_generator(model):
    d, h = TINY.d_model, TINY.ffn_hidden
    E = model.tensor("embed", dtype=torch.float32, shape=(TINY.vocab, d)).cpu().numpy()
    assert np.array_equal(E.astype(np.float64), oracle.embed_table(TINY))
    H = model.tensor("head", dtype=torch.float32, shape=(TINY.vocab, d)).cpu().numpy()
    assert np.array_equal(H.T.astype(np.float64), oracle.head_matrix(TINY))
    for l in range(TINY.n_layers):
        W = oracle.layer_weights(TINY, l)
        qkv = model.tensor("wqkv", l, torch.float32, (3 * d, d)).cpu().numpy().astype(np.float64)
        assert np.array_equal(qkv, np.concatenate([W["wq"].T, W["wk"].T, W["wv"].T]))
        gu = model.tensor("wgu", l, torch.float32, (2 * h, d)).cpu().numpy().astype(np.float64)
        for j in range(h // 128):   # gate/up interleaved in blocks of 128 rows
            assert np.array_equal(gu[256 * j:256 * j + 128], W["wg"].T[128 * j:128 * (j + 1)])
            assert np.array_equal(gu[256 * j + 128:256 * (j + 1)], W["wu"].T[128 * j:128 * (j + 1)])
        wd = model.tensor("wd", l, torch.float32, (d, h)).cpu().numpy().astype(np.float64)
        assert np.array_equal(wd, W["wd"].T)


@pytest.mark.parametrize("B,S", [(1, 32), (1, 1), (3, 17), (2, 64)])
def test_prefill_matches_oracle(model, B, S):
    tok = _tok(B, S)
    lg = model.prefill(torch.from_numpy(tok).cuda()).cpu().numpy()
    ref = oracle.prefill(TINY, tok)
    assert rel_max_err(lg, ref) <= TOL
    greedy_bar(lg, ref, what="tiny fp32 prefill")


def test_kv_cache_holds_rotated_keys_and_plain_values(model):
    B, S = 1, 32
    tok = _tok(B, S)
    model.prefill(torch.from_numpy(tok).cuda(), logits=False)
    _, cache = oracle.prefill(TINY, tok, return_cache=True)
    L, H, hd, smax = TINY.n_layers, TINY.n_heads, TINY.head_dim, 64
    kv = model.tensor("kv", dtype=torch.float32, shape=(L, 2, 3, H, smax, hd)).cpu().numpy()
    for l in range(L):
        k_ref, v_ref = cache[l]
        for which, ref in ((0, k_ref), (1, v_ref)):
            got = kv[l, which, 0, :, :S].astype(np.float64)
            assert np.max(np.abs(got - ref[0])) <= TOL * np.sqrt(np.mean(ref ** 2))


def test_greedy_decode_matches_oracle(model):
    B, S, steps = 2, 20, 8
    tok = _tok(B, S)
    model.prefill(torch.from_numpy(tok).cuda(), logits=False)
    cur = torch.from_numpy(_tok(B, 1, first=1000)[:, 0].copy()).cuda()
    seq = [tok, cur.cpu().numpy()[:, None]]
    logits = []
    for _ in range(steps):
        nxt, lg = model.decode_step(cur)
        logits.append(lg.cpu().numpy())
        cur = nxt
        seq.append(nxt.cpu().numpy()[:, None])
    full = np.concatenate(seq, axis=1)[:, :S + steps]
    ref = oracle.prefill(TINY, full)              # decode == prefill row (pinned in the oracle)
    got = np.stack(logits, axis=1)                # [B, steps, V]
    assert rel_max_err(got, ref[:, S:S + steps]) <= TOL
    # the tokens it chose are the oracle's greedy choices
    assert argmax_agreement(got, ref[:, S:S + steps])[0] == 1.0
    assert model.position == S + steps


def test_generate_equals_repeated_decode_steps(model):
    B, S, steps = 3, 12, 6
    tok = torch.from_numpy(_tok(B, S)).cuda()
    first = torch.from_numpy(_tok(B, 1, first=2000)[:, 0].copy()).cuda()
    model.prefill(tok, logits=False)
    out = model.generate(first, steps).cpu().numpy()
    model.prefill(tok, logits=False)
    cur, seq = first, []
    for _ in range(steps):
        cur, _ = model.decode_step(cur)
        seq.append(cur.cpu().numpy())
    assert np.array_equal(out, np.stack(seq))


def test_decode_past_max_seq_is_rejected(model):
    tok = torch.from_numpy(_tok(1, 64)).cuda()
    model.prefill(tok, logits=False)
    with pytest.raises(lb.LlamaError) as e:
        model.decode_step(tok[:, 0].contiguous())
    assert e.value.code == -5
