"""Host logic of bench.py's per-kernel prefill sweep (no GPU): the sweep
points are the 65B-width grid (batch {1, 8} x length {512, 1024, 2048}),
and the per-family table sums the profiled regions of a family and rates
each against the peak that bounds it."""
import pytest

import bench

PEAKS = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}


def test_sweep_points_are_the_batch_length_grid():
    assert sorted(bench.SWEEP_POINTS) == sorted((b, s) for b in (1, 8) for s in (512, 1024, 2048))


def test_sweep_table_rates_each_family_against_its_bound():
    prof = {
        # two projection regions of one family: 3 ms, 4.2e12 FLOP -> 1400 TFLOP/s
        "prefill_gemm_qkv": dict(ms=1.0, launches=16, calls=16, bytes=1e9, flops=1.2e12),
        "prefill_gemm_gu": dict(ms=2.0, launches=16, calls=16, bytes=2e9, flops=3.0e12),
        # attention: 0.5 ms, 2e11 FLOP -> 400 TFLOP/s
        "prefill_attention": dict(ms=0.5, launches=16, calls=16, bytes=1e8, flops=2e11),
        # memory-bound: 0.1 ms, 3e8 bytes -> 3000 GB/s
        "prefill_rmsnorm": dict(ms=0.1, launches=33, calls=33, bytes=3e8, flops=0.0),
    }
    t = bench.sweep_table(prof, PEAKS)
    g = t["gemm_tc prefill (tcgen05, fused epilogues)"]
    assert g["ms"] == pytest.approx(3.0) and g["launches"] == 32
    assert g["tflops"] == pytest.approx(1400.0) and g["frac_bf16"] == pytest.approx(1400.0 / 1600.0, abs=1e-4)
    a = t["prefill_attention"]
    assert a["tflops"] == pytest.approx(400.0) and "gbs" not in a
    r = t["prefill_rmsnorm"]
    assert r["gbs"] == pytest.approx(3000.0) and r["frac_hbm"] == pytest.approx(0.5) and "tflops" not in r
    # ordered by device time, largest first
    assert list(t)[0] == "gemm_tc prefill (tcgen05, fused epilogues)"


def test_sweep_table_skips_rates_of_unmeasured_regions():
    t = bench.sweep_table({"prefill_argmax": dict(ms=0.0, launches=1, calls=1, bytes=1e6, flops=0.0)}, PEAKS)
    assert t["prefill_argmax"] == dict(ms=0.0, launches=1)
