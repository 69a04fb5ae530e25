"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test names the passage or the mathematical fact it checks.  Together
they are chosen so that a plausible slip in the oracle (a dropped gain or
eps, a wrong sign or pairing in RoPE, a transposed or swapped FFN operand,
a missing mask, a post-norm ordering, a missing parameter tensor) fails at
least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
from scipy.special import expit

import oracle
from synth.workloads import TINY, ModelShape

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- RMSNorm

def test_rmsnorm_worked_example_and_centred_identity():
    """Printed demo: [1,2,3,4] -> x/sqrt(7.5); centred vector equals LayerNorm."""
    g = _golden("rmsnorm_worked_example.json")
    for case in g["cases"]:
        x = np.array(case["x"])
        y = oracle.rms_norm(x, eps=0.0)
        assert np.round(y, g["digits"]).tolist() == case["rms_norm"]
        if "rms_norm_mean" in case:
            assert round(float(y.mean()), 4) == case["rms_norm_mean"]
    # the centred case: RMSNorm output equals the printed LayerNorm output
    c = g["cases"][1]
    y = oracle.rms_norm(np.array(c["x"]), eps=0.0)
    assert np.round(y, 4).tolist() == c["layer_norm"]


def test_rmsnorm_zeros_eps():
    """0/0 is NaN with eps = 0; eps = 1e-5 gives zeros (printed)."""
    z = np.zeros(4)
    with np.errstate(invalid="ignore", divide="ignore"):
        assert np.isnan(oracle.rms_norm(z, eps=0.0)).all()
    assert (oracle.rms_norm(z, eps=1e-5) == 0.0).all()


def test_rmsnorm_closed_forms():
    """eps sits inside the square root; the gain multiplies elementwise; the
    output has unit root-mean-square and is scale invariant (eps = 0)."""
    ones = np.ones(8)
    assert oracle.rms_norm(ones, eps=3.0) == pytest.approx(np.full(8, 0.5), abs=0, rel=1e-15)
    rng = np.random.default_rng(1)
    x = rng.standard_normal((3, 16))
    y = oracle.rms_norm(x, eps=0.0)
    assert np.allclose(np.sqrt((y ** 2).mean(-1)), 1.0, atol=1e-14)
    assert np.allclose(oracle.rms_norm(37.5 * x, eps=0.0), y, atol=1e-14)
    gain = rng.standard_normal(16)
    assert np.allclose(oracle.rms_norm(x, gain, eps=0.0), y * gain, atol=1e-14)
    # no mean subtraction: a constant vector maps to sign(c) * 1
    assert np.allclose(oracle.rms_norm(np.full(5, -2.0), eps=0.0), -1.0)


# ---------------------------------------------------------------- SiLU / SwiGLU

def test_silu_closed_forms():
    assert oracle.silu(np.array(0.0)) == 0.0
    assert oracle.silu(np.array(1.0)) == pytest.approx(1.0 / (1.0 + math.exp(-1.0)), rel=1e-15)
    u = np.linspace(-30, 30, 601)
    assert np.allclose(oracle.silu(u), u * expit(u), rtol=1e-13, atol=1e-300)
    assert oracle.silu(np.array(40.0)) == pytest.approx(40.0, rel=1e-15)
    s = oracle.silu(np.array(-20.0))
    assert s < 0 and abs(s) < 1e-7
    # exact zeros only at 0 (the 0.0% exactly-off units of the SwiGLU demo)
    r = np.random.default_rng(2).standard_normal(100000)
    assert np.count_nonzero(oracle.silu(r) == 0.0) == np.count_nonzero(r == 0.0)


def test_swiglu_brute_force():
    """(SiLU(z Wg) * (z Wu)) Wd, every sum written out as a Python loop."""
    rng = np.random.default_rng(3)
    n, d, h = 3, 4, 5
    z = rng.standard_normal((n, d))
    W = {"wg": rng.standard_normal((d, h)), "wu": rng.standard_normal((d, h)),
         "wd": rng.standard_normal((h, d))}
    ref = np.zeros((n, d))
    for i in range(n):
        for j in range(d):
            acc = 0.0
            for k in range(h):
                g = sum(z[i, m] * W["wg"][m, k] for m in range(d))
                u = sum(z[i, m] * W["wu"][m, k] for m in range(d))
                acc += (g / (1.0 + math.exp(-g))) * u * W["wd"][k, j]
            ref[i, j] = acc
    assert np.allclose(oracle.swiglu_ffn(z, W), ref, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- hidden size, parameter counts

def test_hidden_size_rule():
    """Size table: 4096->11008, 5120->13824, 6656->17920, 8192->22016 (not 10923)."""
    for s in _golden("llama_shapes.json")["sizes"]:
        assert oracle.llama_hidden(s["dim"]) == s["ffn"]
    assert oracle.llama_hidden(128) == 512
    assert TINY.ffn_hidden == oracle.llama_hidden(TINY.d_model)


def _shape(dim, layers, ffn, vocab):
    return ModelShape("t", layers, dim, dim // 128, 128, ffn, vocab)


def test_parameter_counts_from_allocated_shapes():
    """count_params column of the size table, summed over every tensor the
    oracle builds, and the bias=True break (+1,622,016 for 7B)."""
    g = _golden("llama_shapes.json")
    for s in g["sizes"]:
        assert oracle.count_params(_shape(s["dim"], s["layers"], s["ffn"], g["vocab"])) == s["count_params"]
    s7 = _shape(4096, 32, 11008, g["vocab"])
    assert oracle.count_params(s7, bias=True) == g["bias_7b"]["count_params"]
    assert oracle.count_params(s7, bias=True) - oracle.count_params(s7) == g["bias_7b"]["delta"]
    f = g["ffn_d4096"]
    d = 4096
    assert 3 * d * oracle.llama_hidden(d) == f["swiglu_params"]
    assert 3 * d * 4 * d == f["swiglu_4d_params"]
    assert 2 * d * 4 * d == f["relu_4d_params"]
    # inference ~ 2N FLOPs per token
    assert 2 * oracle.count_params(s7) == pytest.approx(g["inference_flops_per_token_7b"], rel=0.005)
    assert oracle.count_params(TINY) == 780928


# ---------------------------------------------------------------- RoPE

def test_rope_special_cases():
    """Pair i = (x[2i], x[2i+1]) turns by p * 10000^(-2i/d): with d = 4 the
    first pair turns by p, the second by p/100; interleaved, not half-split."""
    p = 0.7
    out = oracle.rope(np.array([[1.0, 0.0, 0.0, 0.0]]), np.array([p]))
    assert np.allclose(out, [[math.cos(p), math.sin(p), 0, 0]], atol=1e-15)
    out = oracle.rope(np.array([[0.0, 1.0, 0.0, 0.0]]), np.array([p]))
    assert np.allclose(out, [[-math.sin(p), math.cos(p), 0, 0]], atol=1e-15)
    out = oracle.rope(np.array([[0.0, 0.0, 1.0, 0.0]]), np.array([p]))
    assert np.allclose(out, [[0, 0, math.cos(p / 100), math.sin(p / 100)]], atol=1e-15)
    x = np.random.default_rng(4).standard_normal((3, 6, 32))
    assert np.array_equal(oracle.rope(x, np.zeros(6)), x)          # position 0 = identity


def test_rope_preserves_norm_and_depends_on_offset_only():
    """Each pair is a 2-D rotation (norm preserved); (R_m q).(R_n k) depends
    only on n - m ([NAR] relative-offset identity), and equals q^T R_{n-m} k."""
    rng = np.random.default_rng(5)
    d = 128
    x = rng.standard_normal((7, d))
    pos = np.array([0, 1, 5, 100, 1000, 2047, 4096])
    assert np.allclose(np.linalg.norm(oracle.rope(x, pos), axis=-1), np.linalg.norm(x, axis=-1),
                       rtol=1e-13)
    q, k = rng.standard_normal(d), rng.standard_normal(d)

    def score(m, n):
        return float(oracle.rope(q[None], np.array([m]))[0] @ oracle.rope(k[None], np.array([n]))[0])

    for m, n in [(3, 1), (1, 3), (10, 17), (2000, 5)]:
        assert score(m, n) == pytest.approx(score(m + 91, n + 91), abs=1e-10)
        # q^T R_{n-m} k with R built as a block-diagonal rotation matrix
        theta = 10000.0 ** (-np.arange(0, d, 2) / d)
        R = np.zeros((d, d))
        for i, t in enumerate(theta):
            a = (n - m) * t
            R[2 * i:2 * i + 2, 2 * i:2 * i + 2] = [[math.cos(a), -math.sin(a)], [math.sin(a), math.cos(a)]]
        assert score(m, n) == pytest.approx(float(q @ R @ k), abs=1e-10)
    assert score(3, 1) != pytest.approx(score(3, 0), abs=1e-6)


# ---------------------------------------------------------------- attention

def _attention_loops(q, k, v):
    n, dh = q.shape
    out = np.zeros_like(v)
    for t in range(n):
        s = [sum(q[t, c] * k[j, c] for c in range(dh)) / math.sqrt(dh) for j in range(t + 1)]
        m = max(s)
        w = [math.exp(x - m) for x in s]
        tot = sum(w)
        for c in range(v.shape[1]):
            out[t, c] = sum(w[j] * v[j, c] for j in range(t + 1)) / tot
    return out


def test_attention_brute_force():
    rng = np.random.default_rng(6)
    for n, dh in [(1, 4), (5, 4), (9, 8)]:
        q, k, v = (rng.standard_normal((n, dh)) for _ in range(3))
        assert np.allclose(oracle.causal_attention(q, k, v), _attention_loops(q, k, v),
                           rtol=1e-12, atol=1e-12)


def test_attention_special_cases():
    rng = np.random.default_rng(7)
    n, dh = 6, 8
    q, k, v = (rng.standard_normal((n, dh)) for _ in range(3))
    out = oracle.causal_attention(q, k, v)
    assert np.array_equal(out[0], v[0])                                   # row 0 sees only key 0
    same_k = np.tile(k[:1], (n, 1))                                       # equal keys: running mean
    out2 = oracle.causal_attention(q, same_k, v)
    assert np.allclose(out2, np.cumsum(v, 0) / np.arange(1, n + 1)[:, None], atol=1e-14)
    # causality: later q/k/v rows do not move earlier outputs
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    q2[4:] += 3.0
    k2[4:] -= 2.0
    v2[4:] *= 5.0
    assert np.allclose(oracle.causal_attention(q2, k2, v2)[:4], out[:4], atol=1e-15)


# ---------------------------------------------------------------- block and model

def _small_shape(layers=2):
    return ModelShape("s", layers, 64, 4, 16, oracle.llama_hidden(64), 97, dtype="f32")


def test_pre_norm_block_identity_when_branches_add_nothing():
    """Pre-norm: the trunk is only ever added to.  With Wo = Wd = 0 the block
    returns x exactly (a post-norm block would return norm(x))."""
    s = _small_shape()
    W = oracle.layer_weights(s, 0)
    W["wo"] = np.zeros_like(W["wo"])
    W["wd"] = np.zeros_like(W["wd"])
    x = np.random.default_rng(8).standard_normal((5, s.d_model)) * 3.0
    assert np.array_equal(oracle.block_forward(s, x, weights=W), x)


def test_single_token_attention_reduces_to_value_path():
    """One token: RoPE at position 0 is the identity and the softmax over one
    key is 1, so the attention branch is RMSNorm(x) Wv Wo (not Wq or Wk)."""
    s = _small_shape()
    W = oracle.layer_weights(s, 0)
    W["wd"] = np.zeros_like(W["wd"])
    x = np.random.default_rng(9).standard_normal((1, s.d_model))
    z = x / np.sqrt((x ** 2).mean() + s.norm_eps)
    expect = x + z @ W["wv"] @ W["wo"]
    assert np.allclose(oracle.block_forward(s, x, weights=W), expect, atol=1e-13)


def test_model_invariants_causality_prefix_decode():
    s = _small_shape()
    rng = np.random.default_rng(10)
    tok = rng.integers(0, s.vocab, size=(2, 12))
    lg, cache = oracle.prefill(s, tok, return_cache=True)
    # causality: perturbing tokens after t leaves rows <= t unchanged
    tok2 = tok.copy()
    tok2[:, 7:] = (tok2[:, 7:] + 5) % s.vocab
    assert np.allclose(oracle.prefill(s, tok2)[:, :7], lg[:, :7], atol=1e-12)
    assert not np.allclose(oracle.prefill(s, tok2)[:, 7:], lg[:, 7:])
    # prefix truncation
    assert np.allclose(oracle.prefill(s, tok[:, :5]), lg[:, :5], atol=1e-12)
    # decode (one token at a time with a KV cache) == prefill row
    lg9, c9 = oracle.prefill(s, tok[:, :9], return_cache=True)
    for t in range(9, 12):
        logits, nxt, c9 = oracle.decode_step(s, c9, tok[:, t])
        assert np.allclose(logits, lg[:, t], atol=1e-12)
        assert (nxt == np.argmax(lg[:, t], -1)).all()
    assert c9[0][0].shape == cache[0][0].shape
    assert np.allclose(c9[1][0], cache[1][0], atol=1e-12)


def test_no_position_signal_at_the_bottom():
    """Zero blocks: logits = RMSNorm(E[tok]) Whead; the embedding alone, the
    same token at two positions gives the same logits."""
    s = _small_shape(layers=0)
    tok = np.array([[3, 3, 50]])
    lg = oracle.prefill(s, tok)
    assert np.array_equal(lg[0, 0], lg[0, 1])
    E, Wh = oracle.embed_table(s), oracle.head_matrix(s)
    ref = (E[3] / np.sqrt((E[3] ** 2).mean() + s.norm_eps)) @ Wh
    assert np.allclose(lg[0, 0], ref, atol=1e-14)


# ---------------------------------------------------------------- bf16 storage

def test_round_bf16_is_nearest_even():
    import synth
    x = np.concatenate([synth.normal(0, 5, 5000) * 0.02, synth.normal(0, 6, 500) * 50.0,
                        [1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 1.0 + 2.0 ** -8 + 2.0 ** -30]])
    ref = synth.bf16_bits_to_f64(np.array([synth.f64_to_bf16_bits(v) for v in x], dtype=np.uint16))
    assert np.array_equal(oracle.round_bf16(x), ref)


def test_bf16_kv_cache_alone_moves_deep_logits_past_2e2():
    """Why the bf16 parity bar is derived from the arithmetic: with every
    step exact in fp64 except the KV cache stored in bf16 (as the 7B workload
    specifies), four 7B-width layers already move the logits by more than
    2e-2 RMS (max norm); the exact and bf16-storage oracles bracket what a
    bf16 implementation can reach."""
    from synth.workloads import LLAMA_7B
    import synth
    s = LLAMA_7B.with_(n_layers=4)
    tok = synth.tokens(0, 64, s.vocab).reshape(1, 64)
    cache = {}

    def w(l):
        if l not in cache:
            cache.clear()
            cache[l] = oracle.layer_weights(s, l)
        return cache[l]

    exact = oracle.prefill(s, tok, weights=w)
    kv_only = oracle.prefill(s, tok, weights=w, storage="bf16-kv")
    rms = np.sqrt(np.mean(exact ** 2))
    assert np.max(np.abs(kv_only - exact)) / rms > 2e-2
    assert np.sqrt(np.mean((kv_only - exact) ** 2)) / rms < 2e-2


def test_bf16_storage_alone_moves_one_7b_block_past_2e2():
    """Why the stated 2e-2 max-norm bound is not asserted even for one block:
    one 7B-shaped block on the 1 x 2048 N(0, 1) trunk, exact in fp64 except
    that every value a bf16 workload stores in bf16 is rounded to bf16
    (normalised projection inputs, Q, K, V, attention output, SwiGLU
    activation), already moves both the block output y and its increment
    y - x by more than 2e-2 of their RMS in max norm, while the RMS-norm
    distance stays far below it."""
    from synth.workloads import BLOCK_7B, SEED
    import synth
    S, d = 2048, BLOCK_7B.d_model
    x = synth.normal_f32(SEED, synth.TRUNK, S * d, 1.0).reshape(S, d).astype(np.float64)
    W = oracle.layer_weights(BLOCK_7B, 0)
    exact = oracle.block_forward(BLOCK_7B, x, weights=W)
    stored = oracle.block_forward(BLOCK_7B, x, weights=W, storage="bf16")
    for a, b in ((stored, exact), (stored - x, exact - x)):
        r = np.sqrt(np.mean(b ** 2))
        assert np.max(np.abs(a - b)) / r > 2e-2
        assert np.sqrt(np.mean((a - b) ** 2)) / r < 5e-3


def test_bf16_storage_alone_flips_over_1pct_of_greedy_tokens_at_two_7b_layers():
    """Why strict greedy agreement >= 99 % is not asserted at 7B widths: with
    random-init weights the top two of 32000 logits are often close, and
    bf16 storage alone (everything else exact) already changes the greedy
    token at more than 1 % of the positions of a two-layer 7B-width model.
    The GPU tests hold the GPU to the flip count of bf16 storage instead."""
    from synth.workloads import LLAMA_7B, SEED
    import synth
    s = LLAMA_7B.with_(n_layers=2)
    tok = synth.tokens(SEED, 2 * 256, s.vocab).reshape(2, 256)
    exact, stored = oracle.prefill(s, tok, storage=(None, "bf16"))
    assert np.mean(exact.argmax(-1) == stored.argmax(-1)) < 0.99


# ---------------------------------------------------------------- grouped keys and values

def _gqa_shape(n_kv):
    return ModelShape("gqa", 1, 64, 4, 16, 128, 50, dtype="f32", n_kv_heads=n_kv)


@pytest.mark.parametrize("n_kv", [1, 2])
def test_grouped_kv_equals_mha_with_the_group_columns_repeated(n_kv):
    """[NAR] "GQA Was Not an Original LLaMA Feature": query heads share K/V
    heads.  Reading: query head h uses K/V head floor(h / (H / n_kv)).  The
    same forward pass written as plain multi-head attention, with each query
    head's K/V columns copied from its group's, must give the same logits;
    a wrong group map (h mod n_kv, or the groups of another head) does not."""
    s = _gqa_shape(n_kv)
    mha = s.with_(n_kv_heads=0)
    W = oracle.layer_weights(s, 0)
    G, hd = s.n_heads // n_kv, s.head_dim
    Wm = dict(W)
    for name in ("wk", "wv"):
        Wm[name] = np.concatenate([W[name][:, (h // G) * hd:(h // G + 1) * hd] for h in range(s.n_heads)], axis=1)
    tok = np.random.default_rng(21).integers(0, s.vocab, size=(2, 9))
    a = oracle.prefill(s, tok, weights=lambda l: W)
    b = oracle.prefill(mha, tok, weights=lambda l: Wm)
    assert np.allclose(a, b, rtol=0, atol=1e-12)
    # another grouping (h mod n_kv) is a different model unless it coincides
    if n_kv == 2:
        Wx = dict(W)
        for name in ("wk", "wv"):
            Wx[name] = np.concatenate([W[name][:, (h % n_kv) * hd:(h % n_kv + 1) * hd] for h in range(s.n_heads)],
                                      axis=1)
        assert not np.allclose(a, oracle.prefill(mha, tok, weights=lambda l: Wx), atol=1e-6)
    # the weight shapes count the narrower K and V
    assert oracle.count_params(s) == oracle.count_params(mha) - 2 * s.d_model * (s.n_heads - n_kv) * hd


@pytest.mark.parametrize("n_kv", [1, 2, 4])
def test_grouped_kv_cache_size_and_decode(n_kv):
    """The cache holds 2 L S n_kv d_h values per sequence, the page's
    M_KV = 2 L S n_kv d_h b with b bytes per value; decoding one token at a
    time over it reproduces the prefill rows."""
    s = _gqa_shape(n_kv)
    tok = np.random.default_rng(22).integers(0, s.vocab, size=(3, 10))
    lg, cache = oracle.prefill(s, tok, return_cache=True)
    values = sum(k.size + v.size for k, v in cache)
    assert values == 2 * s.n_layers * 10 * n_kv * s.head_dim * 3
    lg7, c7 = oracle.prefill(s, tok[:, :7], return_cache=True)
    for t in range(7, 10):
        logits, nxt, c7 = oracle.decode_step(s, c7, tok[:, t])
        assert np.allclose(logits, lg[:, t], atol=1e-12)
    assert c7[0][0].shape == (3, n_kv, 10, s.head_dim)


# ---------------------------------------------------------------- the bias variant

def _bias_shape():
    return ModelShape("b", 1, 8, 2, 4, 16, 11, dtype="f32", bias=True)


def _bias_weights(s, **nonzero):
    """Every matrix zero except the named ones; biases and shifts from the generator."""
    W = oracle.layer_weights(s, 0)
    for name in ("wq", "wk", "wv", "wo", "wg", "wu", "wd"):
        W[name] = nonzero.get(name, np.zeros_like(W[name]))
    return W


def test_bias_variant_closed_forms():
    """The page's bias=True count ([PFD] "6.7B parameters, 1T tokens: the
    arithmetic"): every linear layer adds a bias, each in-layer norm a shift.
    With all matrices zero a block is y = x + b_o + b_d (V rows all equal
    b_v average to b_v, which W_o = 0 drops); with W_o = I the value bias
    passes, y = x + b_v + b_o + b_d; with W_q = W_k = 0 the causal weights
    are uniform once b_q = 0, so W_v = W_o = I give h_t = x_t + mean_{j<=t}(rms(x_j) g +
    beta_attn) + b_v + b_o; and W_u = W_d = identity blocks give
    y = h + (SiLU(b_g) * (rms(h) g + beta_ffn + b_u))[:d] + b_d."""
    s = _bias_shape()
    d, h = s.d_model, s.ffn_hidden
    x = np.random.default_rng(30).normal(size=(6, d))
    pos = np.arange(6)
    W = _bias_weights(s)
    y = oracle.pre_norm_block(x, W, pos, s)
    assert np.allclose(y, x + W["bo"] + W["bd"], atol=1e-13)
    W = _bias_weights(s, wo=np.eye(d))
    y = oracle.pre_norm_block(x, W, pos, s)
    assert np.allclose(y, x + W["bv"] + W["bo"] + W["bd"], atol=1e-13)
    eye_du = np.eye(d, h)
    W = _bias_weights(s, wv=np.eye(d), wo=np.eye(d), wu=eye_du, wd=eye_du.T)
    W["bq"] = np.zeros(d)       # q = 0: every score 0 (RoPE would turn b_q and b_k by position)
    y = oracle.pre_norm_block(x, W, pos, s)
    zn = oracle.rms_norm(x, np.ones(d), s.norm_eps) + W["beta_attn"]
    hh = x + np.cumsum(zn, axis=0) / (pos + 1)[:, None] + W["bv"] + W["bo"]
    z2 = oracle.rms_norm(hh, np.ones(d), s.norm_eps) + W["beta_ffn"]
    act = oracle.silu(W["bg"])[None, :] * (z2 @ eye_du + W["bu"][None, :])
    assert np.allclose(y, hh + act @ eye_du.T + W["bd"], atol=1e-12)


def test_bias_variant_with_zero_biases_is_the_original_model():
    s = _bias_shape()
    W = oracle.layer_weights(s, 0)
    for name in ("bq", "bk", "bv", "bo", "bg", "bu", "bd", "beta_attn", "beta_ffn"):
        W[name] = np.zeros_like(W[name])
    tok = np.random.default_rng(31).integers(0, s.vocab, size=(2, 7))
    plain = s.with_(bias=False)
    a = oracle.prefill(s, tok, weights=lambda l: W)
    b = oracle.prefill(plain, tok, weights=lambda l: {k: v for k, v in W.items() if k.startswith(("w", "g"))})
    assert np.allclose(a, b, rtol=0, atol=1e-13)
    # and the biases move it
    assert not np.allclose(a, oracle.prefill(s, tok), atol=1e-6)
    # decode == prefill rows with biases
    lg, cache = oracle.prefill(s, tok[:, :5], return_cache=True)
    full = oracle.prefill(s, tok)
    for t in range(5, 7):
        logits, _, cache = oracle.decode_step(s, cache, tok[:, t])
        assert np.allclose(logits, full[:, t], atol=1e-12)
