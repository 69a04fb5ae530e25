"""Comparison helpers shared by the GPU parity tests.

Two bars are applied to bf16 results, both against the exact fp64 oracle and
both printed in full so a run's log shows how far inside them a result is:

* storage_bar: element-wise distance.  The stated bound for bf16 workloads is
  max|err| <= 2e-2 RMS(ref); the figure is printed for every comparison, but
  bf16 storage of the values the workloads store in bf16 already exceeds it
  at one 7B block and at depth (tests/test_oracle_pins.py:
  test_bf16_storage_alone_moves_one_7b_block_past_2e2,
  test_bf16_kv_cache_alone_moves_deep_logits_past_2e2).  What is asserted is
  that the GPU is no further from the exact answer than that storage moves
  the oracle itself, with an allowance for the GPU's own extra roundings.
* greedy_bar: strict greedy agreement.  The stated >= 99 % is asserted for
  the fp32 workloads.  With bf16 storage it is out of reach: random-init
  logits often have near-equal top tokens, and bf16 storage alone changes
  more than 1 % of greedy tokens already at two 7B-width layers
  (test_bf16_storage_alone_flips_over_1pct_of_greedy_tokens_at_two_7b_layers;
  measured on the GPU runs: 1.7 % at two layers of width 512, 9 % at 32
  layers of 7B).  There the GPU may change no more greedy tokens than bf16
  storage alone does (x1.5 + 3), and both counts are printed.
"""
import numpy as np

STATED_BF16_MAX = 2e-2   # max|err| / RMS(ref) stated for bf16-weight / fp32-accumulate workloads
STATED_AGREEMENT = 0.99  # stated share of positions whose greedy token agrees


def rms(a) -> float:
    return float(np.sqrt(np.mean(np.square(np.asarray(a, dtype=np.float64)))))


def rel_max_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(got - ref)) / rms(ref))


def _rows(a):
    a = np.asarray(a, dtype=np.float64)
    return a.reshape(-1, a.shape[-1])


def argmax_agreement(got, ref):
    """(strict agreement, agreement that also accepts near ties).

    A position counts under the second measure when the GPU's chosen token
    has an oracle logit within 2 * max|err| of the oracle's maximum.  It is
    printed for information only; no test asserts it."""
    got, ref = _rows(got), _rows(ref)
    g = got.argmax(-1)
    r = ref.argmax(-1)
    strict = float(np.mean(g == r))
    err = np.max(np.abs(got - ref))
    ok = ref[np.arange(len(g)), g] >= ref.max(-1) - 2 * err
    return strict, float(np.mean(ok))


def greedy_bar(got, exact, stored=None, what=""):
    """Strict greedy agreement of `got` with the exact oracle.

    Without `stored` (fp32 workloads) strict agreement >= 99 % is asserted.
    With `stored` (the oracle with bf16 storage) the GPU may change at most
    1.5 x as many greedy tokens as bf16 storage alone, plus 3 (the GPU's
    roundings are another draw of the same size: a count of a few tens of
    flips fluctuates by about its square root).  Returns the strict
    agreement."""
    strict, relaxed = argmax_agreement(got, exact)
    n = _rows(exact).shape[0]
    flips = round((1.0 - strict) * n)
    msg = dict(positions=n, strict=round(strict, 4), flips=flips, near_tie_relaxed=round(relaxed, 4))
    if stored is None:
        print(f"greedy agreement {what}:", msg)
        assert strict >= STATED_AGREEMENT, msg
        return strict
    s_strict = float(np.mean(_rows(stored).argmax(-1) == _rows(exact).argmax(-1)))
    s_flips = round((1.0 - s_strict) * n)
    msg.update(bf16_storage_strict=round(s_strict, 4), bf16_storage_flips=s_flips)
    print(f"greedy agreement {what}:", msg)
    assert flips <= 1.5 * s_flips + 3, msg
    return strict


def storage_bar(got, exact, stored, rms_factor=1.25, max_factor=1.5, what=""):
    """Accuracy bar for bf16 workloads, derived from the arithmetic.

    `exact` is the fp64 oracle, `stored` the same oracle rounding every value
    the workload stores in bf16.  The GPU result must be no further from the
    exact answer than `rms_factor` (RMS norm) / `max_factor` (max norm) times
    the distance bf16 storage alone produces.  The GPU makes the same
    roundings at the same points, but in its own accumulation order, so its
    error is another draw of about the same size; the factors leave room for
    the roundings only the GPU makes (softmax weights rounded to bf16 for the
    P.V product, fp32 accumulation order): in RMS norm, extra error up to
    0.75x the storage error in quadrature (sqrt(1.25^2 - 1)); the max norm of
    another draw fluctuates more (measured ratios: RMS 0.90 - 1.04, max
    0.77 - 1.15 over the bf16 tests).  Prints the stated max-norm figure
    beside it.  Returns the numbers."""
    r = rms(exact)
    g = np.asarray(got, dtype=np.float64) - exact
    s = np.asarray(stored, dtype=np.float64) - exact
    out = dict(gpu_rms=rms(g) / r, gpu_max=float(np.max(np.abs(g))) / r,
               bf16_rms=rms(s) / r, bf16_max=float(np.max(np.abs(s))) / r)
    out["rms_ratio"] = out["gpu_rms"] / out["bf16_rms"] if out["bf16_rms"] > 0 else float("inf")
    out["max_ratio"] = out["gpu_max"] / out["bf16_max"] if out["bf16_max"] > 0 else float("inf")
    within = "within" if out["gpu_max"] <= STATED_BF16_MAX else "over"
    print(f"accuracy vs exact oracle {what}: max|err|/RMS(ref) = {out['gpu_max']:.5f} "
          f"({within} the stated {STATED_BF16_MAX:g}); bf16 storage alone {out['bf16_max']:.5f}; "
          f"RMS err {out['gpu_rms']:.5f} vs {out['bf16_rms']:.5f}; ratios rms {out['rms_ratio']:.3f} "
          f"max {out['max_ratio']:.3f}")
    assert out["gpu_rms"] <= rms_factor * out["bf16_rms"], out
    assert out["gpu_max"] <= max_factor * out["bf16_max"], out
    return out
