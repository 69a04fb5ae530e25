"""Host logic of bench.py (no GPU).

* The per-kernel prefill sweep: the sweep points are the 65B-width grid
  (batch {1, 8} x length {512, 1024, 2048}), and the per-family table sums
  the profiled regions of a family and rates each against its bound.
* The roofline block: the dominant kernel is rated from the timed steps'
  own device time, and the block is refused when the per-kernel times add
  up to more than the timed step.
* The DRAM-traffic ratio is used only while the kernel's code (comments and
  layout aside) is the one the counters were taken on.
* The ncu launch-list summary sums launches and device time per kernel.
* The clock record (median SM clock, active throttle reasons), the decode
  step's algorithmic bytes (weights once + K/V rows at the mean length) and
  the per-phase spans of the decode-step timeline."""
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


# ----------------------------------------------------------------------------- roofline block

def _decode_prof():
    # one profiled prefill's regions plus 4 eager, stamped decode steps
    return {
        "prefill_gemm_qkv": dict(ms=20.0, launches=32, calls=32, bytes=1e9, flops=2.6e13),
        "prefill_attention": dict(ms=7.0, launches=32, calls=32, bytes=4e8, flops=4.4e12),
        "decode_step": dict(ms=20.0, launches=4, calls=4, bytes=4 * 17.6e9, flops=4 * 2.7e10),
    }


def test_roofline_rates_the_decode_step_by_the_timed_graph_replays():
    """With the timed steps' decode time, the dominant kernel's achieved rate is the
    algorithmic bytes per step x steps over that time (the eager steps only give shares)."""
    steps, graph_ms, bytes_step = 128, 128 * 3.9, 17.64e9
    out = bench.roofline(_decode_prof(), decode_scale=32.0, peaks=PEAKS, peak_src="test",
                         graph_decode_ms=graph_ms, decode_steps=steps, step_ms=650.0,
                         decode_bytes_per_step=bytes_step)
    assert out["kernel"] == "decode_step" and out["bound"] == "hbm"
    achieved = bytes_step / (3.9e-3) / 1e9
    assert out["achieved"] == pytest.approx(achieved, rel=1e-3)
    assert out["frac"] == pytest.approx(achieved / PEAKS["hbm_gbs"], rel=1e-3)
    assert out["launches_timed"] == steps
    assert out["avg_launch_us"] == pytest.approx(3900.0, rel=1e-6)
    assert sum(out["shares"].values()) == pytest.approx(1.0, abs=1e-3)


def test_roofline_refuses_kernel_times_above_the_timed_step():
    out = bench.roofline(_decode_prof(), decode_scale=32.0, peaks=PEAKS, peak_src="test",
                         graph_decode_ms=128 * 3.9, decode_steps=128, step_ms=100.0,
                         decode_bytes_per_step=17.64e9)
    assert set(out) == {"error"}


def test_roofline_of_a_tensor_bound_step_uses_the_sustained_peak():
    prof = {"prefill_gemm_qkv": dict(ms=10.0, launches=4, calls=4, bytes=1e9, flops=1.3e13),
            "prefill_rmsnorm": dict(ms=0.5, launches=8, calls=8, bytes=3e9, flops=0.0)}
    out = bench.roofline(prof, decode_scale=1.0, peaks=PEAKS, peak_src="test", step_ms=20.0)
    assert out["bound"] == "tensor" and out["peak"] == PEAKS["bf16_tflops_sustained"]
    assert out["achieved"] == pytest.approx(1300.0)
    assert out["traffic"] is None


# ----------------------------------------------------------------------------- code hash, traffic

def test_code_hash_ignores_comments_and_layout_but_not_code(tmp_path):
    a = tmp_path / "a.cu"
    b = tmp_path / "b.cu"
    c = tmp_path / "c.cu"
    a.write_text('int f(int x) {\n  // add one\n  return x + 1; /* the\n result */\n}\nconst char* s = "a // b";\n')
    b.write_text('int f(int x) { return x + 1; }   // other words\nconst char* s = "a // b";\n')
    c.write_text('int f(int x) { return x + 2; }\nconst char* s = "a // b";\n')
    assert bench.code_hash(str(a)) == bench.code_hash(str(b))
    assert bench.code_hash(str(a)) != bench.code_hash(str(c))
    # the text of a string literal counts, comment markers inside it included
    d = tmp_path / "d.cu"
    d.write_text('int f(int x) { return x + 1; }\nconst char* s = "a // c";\n')
    assert bench.code_hash(str(d)) != bench.code_hash(str(a))


def test_traffic_ratio_only_while_the_kernel_is_the_profiled_one(tmp_path, monkeypatch):
    # the committed profile names the committed kernel's hash
    r = bench.decode_step_traffic_ratio()
    assert r is not None and 1.0 <= r < 1.1
    changed = tmp_path / "decode_step.cu"
    changed.write_text(open(bench.STEP_SOURCE).read() + "\nint one_more_symbol;\n")
    monkeypatch.setattr(bench, "STEP_SOURCE", str(changed))
    assert bench.decode_step_traffic_ratio() is None


# ----------------------------------------------------------------------------- ncu launch list

def test_summarize_ncu_sums_launches_per_kernel(tmp_path, capsys):
    csv_text = "\n".join([
        "==PROF== Connected to process 1",
        '"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size","Grid Size",'
        '"Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"',
        '"0","1","python","h","void <unnamed>::decode_step_kernel<16, 128, 0>(StepArgs)","1","7","(256, 1, 1)",'
        '"(148, 1, 1)","0","10.0","Command line profiler metrics","gpu__time_duration.sum","nsecond","4000000"',
        '"1","1","python","h","void <unnamed>::decode_step_kernel<16, 128, 0>(StepArgs)","1","7","(256, 1, 1)",'
        '"(148, 1, 1)","0","10.0","Command line profiler metrics","gpu__time_duration.sum","nsecond","4000000"',
        '"2","1","python","h","void <unnamed>::rmsnorm_kernel<__nv_bfloat16>(float const*)","1","7","(256, 1, 1)",'
        '"(8192, 1, 1)","0","10.0","Command line profiler metrics","gpu__time_duration.sum","usecond","2000"',
    ])
    p = tmp_path / "launches.csv"
    p.write_text(csv_text + "\n")
    bench.summarize_ncu(str(p))
    out = capsys.readouterr().out.splitlines()
    rows = {l.split()[0]: l.split() for l in out[1:]}
    step = [l for l in out if l.startswith("decode_step_kernel")][0].split()
    assert step[-4] == "2" and float(step[-3]) == pytest.approx(8.0) and float(step[-1]) == pytest.approx(0.8)
    norm = [l for l in out if l.startswith("rmsnorm_kernel")][0].split()
    assert norm[-4] == "1" and float(norm[-3]) == pytest.approx(2.0) and float(norm[-1]) == pytest.approx(0.2)
    assert rows["total"][1] == "3" and float(rows["total"][2]) == pytest.approx(10.0)


# ----------------------------------------------------------------------------- clocks, bytes, phases

def test_clock_summary_takes_the_median_and_collects_active_reasons():
    cs = bench.ClockSampler(0)
    cs.tmp.write("1965, 1965, 700.1, Not Active, Not Active, Not Active, Active\n"
                 "1830, 1965, 980.0, Not Active, Not Active, Not Active, Active\n"
                 "1965, 1965, 990.5, Active, Not Active, Not Active, Not Active\n"
                 "[N/A], 1965, 0, Not Active, Not Active, Not Active, Not Active\n")
    out = cs.summary()
    assert out["sm_mhz"] == 1965.0 and out["sm_max_mhz"] == 1965.0 and out["samples"] == 3
    assert out["reasons"] == ["hw_slowdown", "sw_power_cap"]


def test_clock_summary_without_samples_says_unavailable():
    cs = bench.ClockSampler(0)
    assert cs.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}


def test_decode_bytes_of_the_7b_workload():
    """Weights once (2 (L (4 d^2 + 3 d h) + d V) bytes) plus K and V rows at the mean
    length of 128 steps after a 2048-token prompt: 13.21 + 4.43 = 17.64 GB per step."""
    from synth.workloads import LLAMA_7B
    flops, step_bytes = bench.algorithmic_work(LLAMA_7B, 4, 2048, 128)
    d, h, V, L = 4096, 11008, 32000, 32
    weights = 2.0 * (L * (4 * d * d + 3 * d * h) + d * V)
    kv = 2.0 * 2 * L * 4 * (2048 + 64.5) * d
    assert step_bytes == pytest.approx(weights + kv)
    assert weights / 1e9 == pytest.approx(13.21, abs=0.01) and kv / 1e9 == pytest.approx(4.43, abs=0.01)
    n = 4 * 2048
    assert flops == pytest.approx(2.0 * n * (4 * d * d + 3 * d * h) * L + 2.0 * n * d * V
                                  + 2.0 * 4 * 2048 * 2049 * d * L)


def test_step_phases_sum_each_phase_type_over_layers():
    import numpy as np
    L = 2
    P = 3 + 5 * L
    tl = np.zeros((2, P, 2), dtype=np.uint64)
    t = 0
    for p in range(P):          # CTA 0 starts each phase at t, CTA 1 ends it 1000 ns later
        tl[0, p] = (t, t + 1000)
        tl[1, p] = (t + 200, t + 2000)
        t += 2500               # 500 ns gap after every phase
    out = bench.step_phases(tl, L)
    assert out["embed"] == 2.0 and out["head"] == 2.0 and out["argmax"] == 2.0
    for name in ("qkv", "attention", "o_proj", "gate_up", "down"):
        assert out[name] == 4.0           # 2 us per layer, 2 layers
    assert out["barrier_gaps"] == pytest.approx(0.5 * (P - 1))
    assert out["total"] == pytest.approx((2500 * (P - 1) + 2000) / 1e3)
