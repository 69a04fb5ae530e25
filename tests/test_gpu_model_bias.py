"""The bias variant ([PFD] "6.7B parameters, 1T tokens: the arithmetic",
bias=True: every linear layer adds a bias, each in-layer RMSNorm a shift):
prefill and greedy decode against the fp64 oracle with the same biases,
under the derived bf16 storage bar (tests/_parity.storage_bar) or the fp32
1e-4 bound.  The fused decode step folds each norm shift into the consuming
projection's bias (W (g x / rms + beta) + b = W (g x) / rms + (b + W beta)),
so this also checks that reassociation."""
import numpy as np
import pytest
import torch

import decoder_only_b200 as lb
import oracle
import synth
from synth.workloads import LLAMA_7B, ModelShape, SEED, TINY
from _parity import greedy_bar, rms, storage_bar

pytestmark = pytest.mark.gpu


def _run(shape, B, prompt=40, steps=3):
    toks = synth.tokens(SEED + 7, B * (prompt + steps), shape.vocab).reshape(B, prompt + steps)
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
    return np.concatenate([pre, np.stack(dec, axis=1)], axis=1), toks


@pytest.mark.parametrize("shape,B", [
    (ModelShape("bias-hd128", 2, 512, 4, 128, 1536, 2048, bias=True), 3),
    (ModelShape("bias-hd64", 2, 256, 4, 64, 768, 1024, bias=True), 17),
    (ModelShape("bias-gqa2", 2, 512, 4, 128, 1536, 2048, n_kv_heads=2, bias=True), 4),
])
def test_bias_variant_against_oracle(shape, B):
    got, toks = _run(shape, B)
    exact, stored = oracle.prefill(shape, toks, storage=(None, "bf16"))
    storage_bar(got, exact, stored)
    greedy_bar(got, exact, stored)


def test_bias_variant_fp32_within_1e4():
    shape = TINY.with_(bias=True, name="tiny-bias")
    got, toks = _run(shape, 2, prompt=24)
    exact = oracle.prefill(shape, toks)
    err = np.max(np.abs(got - exact))
    assert err <= 1e-4 * rms(exact), (err, rms(exact))


def test_bias_variant_7b_widths_two_layers():
    shape = LLAMA_7B.with_(n_layers=2, bias=True, name="llama-7b-bias-2layer")
    got, toks = _run(shape, 2, prompt=48, steps=2)
    exact, stored = oracle.prefill(shape, toks, storage=(None, "bf16"))
    storage_bar(got, exact, stored)
    greedy_bar(got, exact, stored)
