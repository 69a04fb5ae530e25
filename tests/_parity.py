"""Comparison helpers shared by the GPU parity tests."""
import numpy as np


def rms(a) -> float:
    return float(np.sqrt(np.mean(np.square(np.asarray(a, dtype=np.float64)))))


def rel_max_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(got - ref)) / rms(ref))


def argmax_agreement(got, ref):
    """(strict agreement, agreement that also accepts near ties).

    A position counts under the second measure when the GPU's chosen token
    has an oracle logit within 2 * max|err| of the oracle's maximum: the pages
    do not decide between two near-equal tokens, so either is a correct
    greedy choice within the stated error."""
    got = np.asarray(got, dtype=np.float64).reshape(-1, np.shape(got)[-1])
    ref = np.asarray(ref, dtype=np.float64).reshape(-1, np.shape(ref)[-1])
    g = got.argmax(-1)
    r = ref.argmax(-1)
    strict = float(np.mean(g == r))
    err = np.max(np.abs(got - ref))
    ok = ref[np.arange(len(g)), g] >= ref.max(-1) - 2 * err
    return strict, float(np.mean(ok))
