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


def storage_bar(got, exact, stored, rms_factor=1.5, max_factor=2.0):
    """Accuracy bar for bf16 workloads, derived from the arithmetic.

    `exact` is the fp64 oracle, `stored` the same oracle rounding every value
    the workload stores in bf16.  The GPU result must be no further from the
    exact answer than `rms_factor` (RMS norm) / `max_factor` (max norm) times
    the distance bf16 storage alone produces.  Returns the four numbers."""
    r = rms(exact)
    g = np.asarray(got, dtype=np.float64) - exact
    s = np.asarray(stored, dtype=np.float64) - exact
    out = dict(gpu_rms=rms(g) / r, gpu_max=float(np.max(np.abs(g))) / r,
               bf16_rms=rms(s) / r, bf16_max=float(np.max(np.abs(s))) / r)
    print("accuracy vs exact oracle:", {k: round(v, 5) for k, v in out.items()})
    assert out["gpu_rms"] <= rms_factor * out["bf16_rms"], out
    assert out["gpu_max"] <= max_factor * out["bf16_max"], out
    return out
