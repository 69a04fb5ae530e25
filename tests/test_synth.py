"""The seeded input generator: Philox4x32-10 known answers, Box-Muller
normals, nearest-even rounding into bf16, uniform token ids."""
import json
import os

import numpy as np
from scipy import stats

import synth


def test_philox_known_answers():
    with open(os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.json")) as f:
        kat = json.load(f)
    for c in kat["cases"]:
        ctr = [int(x, 16) for x in c["ctr"]]
        key = [int(x, 16) for x in c["key"]]
        assert [int(x) for x in synth.philox4x32_10(ctr, key)] == [int(x, 16) for x in c["out"]]


def test_normal_draw_is_standard_normal():
    z = synth.normal(0, 12345, 1 << 20)
    n = z.size
    assert abs(z.mean()) < 5 / np.sqrt(n)
    assert abs(z.var() - 1.0) < 5 * np.sqrt(2.0 / n)
    assert stats.kstest(z, "norm").pvalue > 1e-4
    # deterministic, counter addressed: any sub-range reproduces the same values
    assert np.array_equal(synth.normal(0, 12345, 100, first=1000), z[1000:1100])
    assert not np.array_equal(synth.normal(1, 12345, 100), z[:100])


def _nearest_bf16(x):
    """Nearest bf16 by explicit neighbour comparison, ties to even."""
    bits = np.float64(x).view(np.uint64)
    sign = bits & np.uint64(1 << 63)
    mag = bits & ~np.uint64(1 << 63)
    f = np.abs(np.float64(x))
    lo32 = np.float32(f)
    # largest bf16 <= |x|: truncate an fp32 at or below |x|
    if np.float64(lo32) > f:
        lo32 = np.nextafter(lo32, np.float32(0))
    lo = np.uint32(lo32.view(np.uint32) & np.uint32(0xFFFF0000))
    lo_v = np.float64(lo.view(np.float32))
    hi = np.uint32(lo + np.uint32(0x10000))
    hi_v = np.float64(hi.view(np.float32))
    dl, dh = f - lo_v, hi_v - f
    if dl < dh or (dl == dh and ((lo >> np.uint32(16)) & np.uint32(1)) == 0):
        r = lo
    else:
        r = hi
    out = int(r >> np.uint32(16))
    if sign:
        out |= 0x8000
    del mag
    return out


def test_bf16_rounding_is_nearest_even_from_fp64():
    rng = np.random.default_rng(0)
    xs = list(rng.standard_normal(3000) * 0.02) + list(rng.standard_normal(300) * 50)
    # exact ties and values just beside them (double rounding through fp32 would fail these)
    for base in (1.0, 0.015625, 0.0234375):
        b = np.float64(base)
        ulp = b * 2.0 ** -7
        xs += [b + ulp / 2, b + 1.5 * ulp, b + ulp / 2 + 2.0 ** -40 * b, b + ulp / 2 - 2.0 ** -40 * b,
               -(b + ulp / 2)]
    for x in xs:
        assert synth.f64_to_bf16_bits(x) == _nearest_bf16(x), x


def test_stored_values_match_their_dtype():
    z = synth.normal(0, 77, 4096, scale=0.02)
    f32 = synth.normal_stored(0, 77, 4096, 0.02, "f32")
    assert np.array_equal(f32, z.astype(np.float32).astype(np.float64))
    bf = synth.normal_stored(0, 77, 4096, 0.02, "bf16")
    assert np.array_equal(bf, synth.bf16_bits_to_f64(synth.normal_bf16_bits(0, 77, 4096, 0.02)))
    assert np.max(np.abs(bf - z) / np.abs(z)) <= 2.0 ** -8


def test_tokens_uniform_in_range():
    t = synth.tokens(0, 200000, 1000)
    assert t.min() >= 0 and t.max() < 1000
    counts = np.bincount(t, minlength=1000)
    assert stats.chisquare(counts).pvalue > 1e-4
    assert np.array_equal(synth.tokens(0, 10, 1000, first=50), t[50:60])
