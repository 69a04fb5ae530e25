#!/usr/bin/env python
"""Throughput of the LLaMA pre-norm decoder forward pass on B200.

Default workload (one GPU): the LLaMA-7B-shaped model -- 32 layers, d 4096,
32 heads x 128, FFN hidden 11008, vocab 32000, bf16 weights N(0, 0.02^2)
drawn on the device from seed 0 -- running a causal prefill of 4 sequences x
2048 uniform random token ids (logits for every position), then 128 greedy
decode steps over the contiguous bf16 KV cache.  One step is that whole
pass; `value` counts prompt plus generated tokens per second over all ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl b200|reference]

Under torchrun every rank runs an independent replica (no collective on the
data path: sequences are independent); the timed region is bracketed by a
barrier and a device synchronise, and the time is the max over ranks.

--impl reference times the fp64 CPU oracle on the host cores on a bounded
sample of the same workload (rank 0 only) and prints the same JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "LLaMA-shape tokens/s (prefill, decode) on 1 B200; % of BF16/HBM roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

WORKLOADS = {
    "7b": dict(model="LLAMA_7B", batch=4, seq=2048, decode=128,
               desc="llama-7b: prefill 4 x 2048 (logits at every position) + 128 greedy decode steps"),
    "13b-decode": dict(model="LLAMA_13B", batch=32, seq=2048, decode=256,
                       desc="llama-13b: 256 greedy decode steps, batch 32, 2048-token prompts prefilled untimed"),
    "65b-slice": dict(model="LLAMA_65B_SLICE", batch=8, seq=2048, decode=0,
                      desc="llama-65b widths, 16 layers: prefill 8 x 2048 (logits at every position)"),
    "33b": dict(model="LLAMA_33B", batch=4, seq=2048, decode=128,
                desc="llama-33b: prefill 4 x 2048 (logits at every position) + 128 greedy decode steps"),
    # small case of the 7B kernels (same shapes per launch) for ncu captures
    "7b-2layer": dict(model="LLAMA_7B", layers=2, batch=4, seq=2048, decode=128,
                      desc="llama-7b widths, 2 layers: prefill 4 x 2048 + 128 greedy decode steps"),
}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS if k in d}, "measured (MEASURED_PEAKS.json)"
    return dict(FALLBACK_PEAKS), "fallback (no MEASURED_PEAKS.json)"


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampled every 200 ms while running."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=self.tmp, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        self.tmp.flush()
        with open(self.tmp.name) as f:
            rows = [r.split(",") for r in f.read().strip().splitlines() if r.strip()]
        os.unlink(self.tmp.name)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm, mx, reasons = [], [], set()
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 7:
                continue
            try:
                sm.append(float(r[0]))
                mx.append(float(r[1]))
            except ValueError:
                continue
            for n, v in zip(names, r[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- helpers

def algorithmic_work(shape, B, S, steps):
    """FLOPs of one prefill (causal attention halved) and bytes of one decode
    step (every weight once + the KV cache read + activations), average over
    the decode steps."""
    d, h, V, L = shape.d_model, shape.ffn_hidden, shape.vocab, shape.n_layers
    n = B * S
    gemm = 2.0 * n * (4 * d * d + 3 * d * h) * L + 2.0 * n * d * V
    attn = 2.0 * B * S * (S + 1) * d * L
    wbytes = 2.0 * (L * (4 * d * d + 3 * d * h) + d * V)
    mean_len = S + (steps + 1) / 2.0
    kv = 2.0 * 2 * L * B * mean_len * d
    return gemm + attn, wbytes + kv


PHASE_NAMES = ["embed", "qkv", "attention", "o_proj", "gate_up", "down", "head", "argmax"]


def step_phases(tl, n_layers):
    """Per phase type of the fused decode step: summed critical-path time
    (first start to last end over the CTAs) and the barrier gaps after each
    phase (last end to the next phase's first start), in microseconds."""
    import numpy as np
    start = tl[:, :, 0].astype(np.float64)
    end = tl[:, :, 1].astype(np.float64)
    P = tl.shape[1]
    s0, e1 = start.min(0), end.max(0)
    out = {n: 0.0 for n in PHASE_NAMES}
    gaps = 0.0
    for p in range(P):
        if p == 0:
            name = "embed"
        elif p - 1 < 5 * n_layers:
            name = PHASE_NAMES[1 + (p - 1) % 5]
        else:
            name = "head" if p - 1 == 5 * n_layers else "argmax"
        out[name] += (e1[p] - s0[p]) / 1e3
        if p + 1 < P:
            gaps += (s0[p + 1] - e1[p]) / 1e3
    res = {k: round(v, 1) for k, v in out.items()}
    res["barrier_gaps"] = round(gaps, 1)
    res["total"] = round((e1[-1] - s0[0]) / 1e3, 1)
    return res


def kernel_family(region: str) -> str:
    if region.startswith("prefill_gemm"):
        return "gemm_tc prefill (tcgen05, fused epilogues)"
    if region.startswith("decode_gemm"):
        return "gemm_tc decode (tcgen05 swap-AB split-K)"
    return region


TRAFFIC_PROFILE = os.path.join(ROOT, "profiles", "decode_step_llama7b_2layer_dram.md")
STEP_SOURCE = os.path.join(ROOT, "decoder_only_b200", "csrc", "decode_step.cu")


def code_hash(path: str) -> str:
    """sha256 (16 hex digits) of a C++/CUDA source with its comments and
    whitespace removed: it changes when the code does, not its comments."""
    import hashlib
    with open(path) as f:
        src = f.read()
    out, i, n = [], 0, len(src)
    while i < n:
        if src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        elif src[i] == '"':                      # string literal: kept as is
            j = i + 1
            while j < n and src[j] != '"':
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        else:
            out.append(src[i])
            i += 1
    return hashlib.sha256("".join("".join(out).split()).encode()).hexdigest()[:16]


def decode_step_traffic_ratio():
    """DRAM traffic / algorithmic bytes of the fused decode step from the
    committed ncu summary, or None when the kernel's code has changed since
    the counters were taken."""
    try:
        with open(TRAFFIC_PROFILE) as f:
            txt = f.read()
        h = code_hash(STEP_SOURCE)
    except OSError:
        return None
    ratio = re.search(r"traffic_ratio:\s*([0-9.]+)", txt)
    src = re.search(r"kernel_code_sha256_16:\s*([0-9a-f]+)", txt)
    if not ratio or not src or src.group(1) != h:
        return None
    return float(ratio.group(1))


def roofline(prof, decode_scale, peaks, peak_src, graph_decode_ms=None, decode_steps=0, step_ms=None,
             decode_bytes_per_step=None):
    """Dominant kernel over one step.

    Prefill kernels: the live per-region timing of one profiled (eager)
    prefill.  The fused decode step (one kernel per step, replayed from a
    CUDA graph in the timed region): with `graph_decode_ms` (the timed
    steps' decode time, CUDA events around the graph replays) its time per
    launch is graph_decode_ms / decode_steps and its algorithmic bytes per
    launch `decode_bytes_per_step` (weights once + the K and V rows at the
    mean cache length of the timed steps); the eager, stamped profiled steps
    give only the other kernels' shares.  The block is
    refused (returned as an error note) when the per-kernel times add up to
    more than the timed step `step_ms`."""
    fam = {}
    for name, e in prof.items():
        scale = decode_scale if name.startswith("decode") else 1.0
        f = fam.setdefault(kernel_family(name), dict(ms=0.0, bytes=0.0, flops=0.0, launches=0, step_ms=0.0))
        f["ms"] += e["ms"]
        f["bytes"] += e["bytes"]
        f["flops"] += e["flops"]
        f["launches"] += e["launches"]
        f["step_ms"] += e["ms"] * scale
    timing = "eager per-region CUDA events (one profiled prefill)"
    if graph_decode_ms is not None and "decode_step" in fam and decode_steps:
        f = fam["decode_step"]
        per = max(f["launches"], 1)
        f["bytes"] = (decode_bytes_per_step if decode_bytes_per_step else f["bytes"] / per) * decode_steps
        f["flops"] = f["flops"] / per * decode_steps
        f["ms"], f["launches"], f["step_ms"] = graph_decode_ms, decode_steps, graph_decode_ms
        timing += "; decode_step: CUDA events around the timed steps' graph replays"
    total = sum(f["step_ms"] for f in fam.values())
    if step_ms is not None and total > 1.02 * step_ms:
        return dict(error=f"per-kernel times add up to {total:.2f} ms, more than the timed step "
                          f"({step_ms:.2f} ms): not reported")
    name, f = max(fam.items(), key=lambda kv: kv[1]["step_ms"])
    per_launch_ms = f["ms"] / max(f["launches"], 1)
    if name.startswith("gemm_tc prefill") or name == "prefill_attention":
        achieved = f["flops"] / (f["ms"] * 1e-3) / 1e12
        peak = peaks["bf16_tflops_sustained"]
        out = dict(bound="tensor", unit="TFLOP/s", peak_kind="bf16 dense, sustained (kernel timed inside a long step)")
    else:
        achieved = f["bytes"] / (f["ms"] * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        out = dict(bound="hbm", unit="GB/s", peak_kind="HBM copy bandwidth")
    traffic = None
    if name == "decode_step":
        r = decode_step_traffic_ratio()
        if r is not None:   # bytes per launch: measured ratio x this launch's algorithmic bytes
            traffic = round(r * f["bytes"] / max(f["launches"], 1))
    out.update(kernel=name, achieved=round(achieved, 1), peak=peak, frac=round(achieved / peak, 4),
               peak_source=peak_src, traffic=traffic, timing=timing, launches_timed=f["launches"],
               avg_launch_us=round(per_launch_ms * 1e3, 2), share_of_step=round(f["step_ms"] / total, 4),
               shares={k: round(v["step_ms"] / total, 4) for k, v in sorted(fam.items(), key=lambda kv: -kv[1]["step_ms"])},
               est_ms_per_step={k: round(v["step_ms"], 2) for k, v in sorted(fam.items(), key=lambda kv: -kv[1]["step_ms"])})
    return out


# ----------------------------------------------------------------------------- CPU oracle

def oracle_sample(shape, B, S, steps, prompt=64, layers=2):
    """Times the fp64 oracle as it stands on a bounded sample of the workload
    and scales it to one full step.  Weights are drawn before timing."""
    import numpy as np
    import oracle
    import synth
    from threadpoolctl import threadpool_info

    sub = shape.with_(n_layers=layers)
    W = [oracle.layer_weights(shape, l) for l in range(layers)]
    tok = synth.tokens(0, prompt + 2, shape.vocab).reshape(1, prompt + 2)
    t0 = time.perf_counter()
    _, cache = oracle.prefill(sub, tok[:, :prompt], weights=lambda l: W[l], return_cache=True)
    t1 = time.perf_counter()
    oracle.decode_step(sub, cache, tok[:, prompt], weights=lambda l: W[l])
    t2 = time.perf_counter()
    # the oracle's head is included in both calls; scale the layers to L
    scale = shape.n_layers / layers
    t_pre_tok = (t1 - t0) * scale / prompt
    t_dec_tok = (t2 - t1) * scale
    step_s = B * S * t_pre_tok + B * steps * t_dec_tok
    value = (B * S + B * steps) / step_s
    threads = max([p.get("num_threads", 1) for p in threadpool_info()] + [1])
    sample = (f"oracle prefill of 1 x {prompt} tokens and one decode step through {layers} of "
              f"{shape.n_layers} layers (+ head), per-token times scaled by {scale:g} in layer count "
              f"to one step of {B}x{S} prefill + {B}x{steps} decode tokens")
    return dict(value=round(value, 4), unit=UNIT, cores=threads, kind="oracle", sample=sample,
                seconds=round(t2 - t0, 3)), step_s


# ----------------------------------------------------------------------------- replicas

def max_over_ranks(x: float, world: int, device="cpu") -> float:
    """The largest of every rank's value (device time of the same region);
    every rank takes this collective step."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(world: int, tokens_per_step: int, steps: int, ms: float) -> float:
    """Whole-job tokens/s: every replica processes tokens_per_step per step;
    the slowest rank's time bounds the job."""
    return world * tokens_per_step * steps / (ms * 1e-3)


def replica_tokens(shape, rank: int, B: int, S: int):
    """Prompt token ids of one replica: each rank its own seeded draw."""
    import synth
    return synth.tokens(synth.workloads.SEED + rank, B * S, shape.vocab).reshape(B, S)


# ----------------------------------------------------------------------------- arms

def run_reference(args, wl, shape):
    import torch.distributed as dist  # noqa: F401
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    B, S, steps = wl["batch"], wl["seq"], wl["decode"]
    vals = []
    for i in range(args.warmup + args.steps):
        cb, step_s = oracle_sample(shape, B, S, steps)
        if i >= args.warmup:
            vals.append((cb["value"], step_s))
    value = statistics.median(v for v, _ in vals)
    ms = statistics.median(s for _, s in vals) * 1e3
    cb["value"] = round(value, 4)
    line = dict(impl="reference", metric=METRIC, value=round(value, 4), unit=UNIT, n_gpus=args.gpus,
                steps=args.steps, warmup=args.warmup, ms_per_step=round(ms, 1), higher_is_better=True,
                scaling="weak", vs_baseline=None, dtype="f64", data="synthetic",
                config=dict(workload=wl["desc"], batch=B, seq_len=S, decode_steps=steps),
                cpu_baseline=cb, e2e=dict(value=round(value, 4), unit=UNIT, h2d_bytes_per_step=0,
                                          d2h_bytes_per_step=0))
    print(json.dumps(line), flush=True)


def run_b200(args, wl, shape):
    import torch
    import torch.distributed as dist

    import decoder_only_b200 as lb
    import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    B, S, steps = wl["batch"], wl["seq"], wl["decode"]
    max_seq = S + steps
    model = lb.Model(shape, max_batch=B, max_seq=max_seq, seed=synth.workloads.SEED)
    tok_host = torch.from_numpy(replica_tokens(shape, rank, B, S))
    tok_host = tok_host.pin_memory()
    tok_dev = tok_host.cuda()
    logits = torch.empty(B, S, shape.vocab, dtype=torch.float32, device="cuda") if wl["name"] != "13b-decode" else None
    gen = torch.empty(max(steps, 1), B, dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream()

    decode_only = wl["name"] == "13b-decode"
    if decode_only:
        model.prefill(tok_dev, logits=False)               # untimed: the prompt cache
        first = tok_dev[:, -1].contiguous()

    def step():
        if decode_only:
            model.rewind(S)
            model.generate(first, steps, out=gen)
        else:
            model.prefill(tok_dev, out=logits)
            if steps:
                model.generate(None, steps, out=gen, batch=B)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if args.ncu:
        for _ in range(args.steps):
            torch.cuda.nvtx.range_push("timed_step")
            step()
            torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize()
        model.close()
        return

    # ------------------------------------------------ timed region (device events)
    # events on the launching stream: one before the first step, and per step
    # one after its prefill and one after its decode steps (graph replays),
    # so that the prefill / decode split comes from the timed steps themselves
    ev0 = torch.cuda.Event(enable_timing=True)
    ev_mid = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev_end = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]

    def timed_step(i):
        if decode_only:
            model.rewind(S)
            ev_mid[i].record(st)
            model.generate(first, steps, out=gen)
        else:
            model.prefill(tok_dev, out=logits)
            ev_mid[i].record(st)
            if steps:
                model.generate(None, steps, out=gen, batch=B)
        ev_end[i].record(st)

    barrier()
    torch.cuda.synchronize()
    l0 = lb.kernel_launches()
    with ClockSampler(local) as clk:
        ev0.record(st)
        for i in range(args.steps):
            timed_step(i)
        torch.cuda.synchronize()
    barrier()
    launches = lb.kernel_launches() - l0
    ms = max_over_ranks(ev0.elapsed_time(ev_end[-1]), world, "cuda")
    clocks = clk.summary()
    tokens_step = (0 if decode_only else B * S) + B * steps
    value = replica_throughput(world, tokens_step, args.steps, ms)

    # ------------------------------------------------ prefill / decode split (same events)
    starts = [ev0] + ev_end[:-1]
    pre = [a.elapsed_time(b) for a, b in zip(starts, ev_mid)]
    dec = [a.elapsed_time(b) for a, b in zip(ev_mid, ev_end)]
    split = dict(prefill_ms=0.0 if decode_only else statistics.median(pre),
                 decode_ms=statistics.median(dec) if steps else 0.0)

    # ------------------------------------------------ end to end from host buffers
    out_host = torch.empty(max(steps, 1), B, dtype=torch.int32).pin_memory()
    e2e_ms = None
    if not decode_only:
        model.complete(tok_host, steps, logits=logits, out_host=out_host)
        torch.cuda.synchronize()
        ee = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        barrier()
        torch.cuda.synchronize()
        ee[0].record(st)
        for _ in range(args.steps):
            model.complete(tok_host, steps, logits=logits, out_host=out_host)
        ee[1].record(st)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = max_over_ranks(ee[0].elapsed_time(ee[1]), world, "cuda")

    # ------------------------------------------------ live per-region timing (roofline)
    peaks, peak_src = load_peaks()
    prof_steps = min(steps, 16)
    lb.profile_reset()
    lb.profile_enable(True)
    if decode_only:
        model.rewind(S)
        model.generate(first, prof_steps, out=gen)
    else:
        model.prefill(tok_dev, out=logits)
        if steps:
            model.generate(None, prof_steps, out=gen, batch=B)
    torch.cuda.synchronize()
    prof = lb.profile_read()
    lb.profile_enable(False)
    flops_pre, bytes_dec = algorithmic_work(shape, B, S, steps)
    roof = roofline(prof, steps / max(prof_steps, 1), peaks, peak_src,
                    graph_decode_ms=split["decode_ms"] if steps and shape.dtype == "bf16" else None,
                    decode_steps=steps, step_ms=ms / args.steps, decode_bytes_per_step=bytes_dec)
    phases = None
    if shape.dtype == "bf16" and steps:
        phases = step_phases(model.step_timeline(), shape.n_layers)

    if rank == 0:
        line = dict(
            metric=METRIC, value=round(value, 2), unit=UNIT, n_gpus=world, steps=args.steps, warmup=args.warmup,
            ms_per_step=round(ms / args.steps, 3), higher_is_better=True, scaling="weak", vs_baseline=None,
            dtype="bf16", data="synthetic (seeded token ids; random-init weights N(0, 0.02^2) drawn on device)",
            config=dict(workload=wl["desc"], model=shape.name, global_batch=B * world, seq_len=S,
                        decode_steps=steps, parallelism=f"replicas x{world}" if world > 1 else "single GPU",
                        l2="inputs larger than L2: every step streams all weights (13+ GB) from HBM"),
            gpu_launches=launches, clocks=clocks, roofline=roof)
        if split["prefill_ms"] > 0:
            pre_s = split["prefill_ms"] * 1e-3
            line["prefill"] = dict(tokens_per_s=round(B * S / pre_s, 1), ms=round(split["prefill_ms"], 3),
                                   tflops=round(flops_pre / pre_s / 1e12, 1),
                                   frac_bf16=round(flops_pre / pre_s / 1e12 / peaks["bf16_tflops_sustained"], 4))
        if steps:
            dec_s = split["decode_ms"] * 1e-3
            line["decode"] = dict(tokens_per_s=round(B * steps / dec_s, 1),
                                  ms_per_step=round(split["decode_ms"] / steps, 4),
                                  gbs=round(bytes_dec * steps / dec_s / 1e9, 1),
                                  frac_hbm=round(bytes_dec * steps / dec_s / 1e9 / peaks["hbm_gbs"], 4))
        if phases:
            line["decode_step_phases_us"] = phases
        if e2e_ms is not None:
            line["e2e"] = dict(value=round(replica_throughput(world, tokens_step, args.steps, e2e_ms), 2), unit=UNIT,
                               h2d_bytes_per_step=B * S * 4, d2h_bytes_per_step=B * steps * 4)
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"], _ = oracle_sample(shape, B, S, steps)
        print(json.dumps(line), flush=True)
    model.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# ----------------------------------------------------------------------------- tensor parallel

def run_tp(args, wl, shape):
    """--parallel tp under torchrun: one model split over the N ranks
    (llama_config.tp_size = N), its prefill's two exchanges per block done by
    NCCL all-reduce (torch.distributed) on the library's exchange stream.
    Decoding is not sharded, so a step is the prefill alone (logits at every
    position); total work is fixed as N grows (scaling "strong")."""
    import datetime

    import torch
    import torch.distributed as dist

    import decoder_only_b200 as lb
    import synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                            device_id=torch.device("cuda", local))
    B, S = wl["batch"], wl["seq"]
    model = lb.Model(shape, max_batch=B, max_seq=S, seed=synth.workloads.SEED, tp=(rank, world))
    model.set_allreduce(lb.dist_allreduce(), chunks=args.tp_chunks)
    tok = torch.from_numpy(replica_tokens(shape, 0, B, S)).cuda()    # every shard sees the same batch
    logits = torch.empty(B, S, shape.vocab, dtype=torch.float32, device="cuda")
    st = torch.cuda.current_stream()
    for _ in range(args.warmup):
        model.prefill(tok, out=logits)
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    dist.barrier()
    torch.cuda.synchronize()
    l0 = lb.kernel_launches()
    with ClockSampler(local) as clk:
        ev[0].record(st)
        for _ in range(args.steps):
            model.prefill(tok, out=logits)
        ev[1].record(st)
        torch.cuda.synchronize()
    dist.barrier()
    launches = lb.kernel_launches() - l0
    ms = max_over_ranks(ev[0].elapsed_time(ev[1]), world, "cuda")
    flops, _ = algorithmic_work(shape, B, S, 0)
    if rank == 0:
        peaks, peak_src = load_peaks()
        per_s = ms * 1e-3 / args.steps
        print(json.dumps(dict(
            metric=METRIC, value=round(B * S * args.steps / (ms * 1e-3), 2), unit=UNIT, n_gpus=world,
            steps=args.steps, warmup=args.warmup, ms_per_step=round(ms / args.steps, 3), higher_is_better=True,
            scaling="strong", vs_baseline=None, dtype="bf16",
            data="synthetic (seeded token ids; random-init weights N(0, 0.02^2) drawn on device)",
            config=dict(workload=f"{wl['desc'].split(':')[0]}: prefill {B} x {S} (logits at every position), "
                                 f"tensor parallel over {world} GPUs", model=shape.name, global_batch=B, seq_len=S,
                        parallelism=f"tp{world} (NCCL all-reduce after O and down, {args.tp_chunks} row blocks)",
                        l2="inputs larger than L2: every step streams all weights from HBM"),
            gpu_launches=launches, clocks=clk.summary(),
            prefill=dict(tflops=round(flops / per_s / 1e12, 1),
                         frac_bf16_per_gpu=round(flops / per_s / 1e12 / world / peaks["bf16_tflops_sustained"], 4),
                         peak_source=peak_src))), flush=True)
    model.close()
    dist.barrier()
    dist.destroy_process_group()


# ----------------------------------------------------------------------------- per-kernel sweep

# (batch, sequence length) points of the per-kernel prefill sweep at the 65B
# widths: seq in {512, 1024, 2048} x batch in {1, 8}
SWEEP_POINTS = [(b, s) for b in (1, 8) for s in (512, 1024, 2048)]


def sweep_table(prof, peaks):
    """Per kernel family of one profiled prefill: device time, launches, and
    the achieved rate against the measured peak that bounds it (tensor
    FLOP/s for the projections and attention, HBM bytes/s for the rest)."""
    fam = {}
    for name, e in prof.items():
        f = fam.setdefault(kernel_family(name), dict(ms=0.0, flops=0.0, bytes=0.0, launches=0))
        f["ms"] += e["ms"]
        f["flops"] += e["flops"]
        f["bytes"] += e["bytes"]
        f["launches"] += e["launches"]
    out = {}
    for k, f in sorted(fam.items(), key=lambda kv: -kv[1]["ms"]):
        r = dict(ms=round(f["ms"], 3), launches=f["launches"])
        if f["ms"] > 0 and f["flops"] > 0 and (k.startswith("gemm_tc prefill") or k == "prefill_attention"):
            t = f["flops"] / (f["ms"] * 1e-3) / 1e12
            r.update(tflops=round(t, 1), frac_bf16=round(t / peaks["bf16_tflops"], 4))
        elif f["ms"] > 0 and f["bytes"] > 0:
            g = f["bytes"] / (f["ms"] * 1e-3) / 1e9
            r.update(gbs=round(g, 1), frac_hbm=round(g / peaks["hbm_gbs"], 4))
        out[k] = r
    return out


def run_sweep(args, wl, shape):
    """Prefill of every SWEEP_POINTS (batch, length) on one model: whole-
    prefill time (CUDA events over --steps runs after --warmup) and one
    profiled prefill split per kernel family.  One JSON line."""
    import torch

    import decoder_only_b200 as lb
    import synth

    torch.cuda.set_device(0)
    bmax = max(b for b, _ in SWEEP_POINTS)
    smax = max(s for _, s in SWEEP_POINTS)
    model = lb.Model(shape, max_batch=bmax, max_seq=smax, seed=synth.workloads.SEED)
    peaks, peak_src = load_peaks()
    st = torch.cuda.current_stream()
    points = []
    for B, S in SWEEP_POINTS:
        tok = torch.from_numpy(synth.tokens(synth.workloads.SEED, B * S, shape.vocab).reshape(B, S)).cuda()
        logits = torch.empty(B, S, shape.vocab, dtype=torch.float32, device="cuda")
        for _ in range(args.warmup):
            model.prefill(tok, out=logits)
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        ev[0].record(st)
        for _ in range(args.steps):
            model.prefill(tok, out=logits)
        ev[1].record(st)
        torch.cuda.synchronize()
        ms = ev[0].elapsed_time(ev[1]) / args.steps
        lb.profile_reset()
        lb.profile_enable(True)
        model.prefill(tok, out=logits)
        torch.cuda.synchronize()
        prof = lb.profile_read()
        lb.profile_enable(False)
        flops, _ = algorithmic_work(shape, B, S, 0)
        tf = flops / (ms * 1e-3) / 1e12
        points.append(dict(batch=B, seq=S, prefill_ms=round(ms, 3), tokens_per_s=round(B * S / (ms * 1e-3), 1),
                           tflops=round(tf, 1), frac_bf16=round(tf / peaks["bf16_tflops_sustained"], 4),
                           kernels=sweep_table(prof, peaks)))
        del logits
    grid = "batch {%s} x length {%s}" % (", ".join(str(b) for b in sorted({b for b, _ in SWEEP_POINTS})),
                                        ", ".join(str(s) for s in sorted({s for _, s in SWEEP_POINTS})))
    print(json.dumps(dict(metric="per-kernel prefill sweep", unit="ms / TFLOP/s / GB/s",
                          workload=wl["desc"].split(":")[0] + ": prefill at every point of " + grid,
                          model=shape.name, steps=args.steps, warmup=args.warmup, peak_source=peak_src,
                          data="synthetic (seeded token ids; random-init weights N(0, 0.02^2) drawn on device)",
                          points=points)), flush=True)
    model.close()


def summarize_ncu(path):
    """Per-kernel launches, total device time and share from an ncu
    `--metrics gpu__time_duration.sum --csv` launch list."""
    import csv
    import re
    with open(path) as f:
        lines = f.read().splitlines()
    start = next(i for i, l in enumerate(lines) if l.startswith('"ID"'))
    rows = list(csv.DictReader(lines[start:]))
    agg = {}
    for r in rows:
        if r.get("Metric Name") != "gpu__time_duration.sum":
            continue
        name = r["Kernel Name"]
        name = re.sub(r"\(.*", "", name)
        m = re.search(r"(gemm_tc_kernel|attn_\w+|\w+_kernel)(<[^>]*>)?", r["Kernel Name"])
        key = m.group(0) if m else name
        v = float(r["Metric Value"].replace(",", ""))
        unit = r.get("Metric Unit", "nsecond")
        scale = {"nsecond": 1e-3, "usecond": 1.0, "msecond": 1e3, "second": 1e6}.get(unit, 1e-3)
        a = agg.setdefault(key, [0, 0.0])
        a[0] += 1
        a[1] += v * scale
    total = sum(v[1] for v in agg.values())
    print(f"{'kernel':70s} {'launches':>9s} {'total_ms':>10s} {'avg_us':>9s} {'share':>7s}")
    for k, (n, us) in sorted(agg.items(), key=lambda kv: -kv[1][1]):
        print(f"{k[:70]:70s} {n:9d} {us / 1e3:10.3f} {us / n:9.2f} {us / total:7.4f}")
    print(f"{'total':70s} {sum(v[0] for v in agg.values()):9d} {total / 1e3:10.3f}")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--workload", default=None, choices=sorted(WORKLOADS),
                    help="default: 7b (65b-slice with --sweep)")
    ap.add_argument("--sweep", action="store_true",
                    help="per-kernel prefill sweep over batch {1, 8} x length {512, 1024, 2048} "
                         "(one JSON line; 1 GPU)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kv-heads", type=int, default=0,
                    help="grouped keys and values: the workload's model with this many key/value heads")
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch")
    ap.add_argument("--parallel", default="replicas", choices=["replicas", "tp"],
                    help="N > 1: independent replicas (default) or one model split over the N GPUs "
                         "(tensor parallel prefill, under torchrun)")
    ap.add_argument("--tp-chunks", type=int, default=4, help="row blocks per exchange with --parallel tp")
    ap.add_argument("--ncu", action="store_true",
                    help="only the warm-up and timed steps, each timed step in an NVTX range 'timed_step' "
                         "(for: ncu --nvtx --nvtx-include timed_step/ ...); prints no JSON")
    ap.add_argument("--summarize-ncu", metavar="CSV",
                    help="print the per-kernel launches / time / share table of an ncu --csv launch list")
    args = ap.parse_args()
    if args.summarize_ncu:
        summarize_ncu(args.summarize_ncu)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    from synth import workloads as wls
    name = args.workload or ("65b-slice" if args.sweep else "7b")
    wl = dict(WORKLOADS[name], name=name)
    shape = getattr(wls, wl["model"])
    if "layers" in wl:
        shape = shape.with_(n_layers=wl["layers"], name=f"{shape.name}-{wl['layers']}layer")
    if args.kv_heads:
        shape = shape.with_(n_kv_heads=args.kv_heads, name=f"{shape.name}-kv{args.kv_heads}")
        wl["desc"] = wl["desc"].replace(":", f" ({args.kv_heads} key/value heads):", 1)
    if args.batch:
        wl["desc"] = wl["desc"].replace(f"{wl['batch']} x", f"{args.batch} x", 1).replace(
            f"batch {wl['batch']}", f"batch {args.batch}", 1)
        wl["batch"] = args.batch
    if args.sweep:
        if args.impl == "reference" or int(os.environ.get("WORLD_SIZE", "1")) > 1:
            ap.error("--sweep times this library on one GPU")
        run_sweep(args, wl, shape)
    elif args.impl == "reference":
        run_reference(args, wl, shape)
    elif args.parallel == "tp":
        if int(os.environ.get("WORLD_SIZE", "1")) < 2:
            ap.error("--parallel tp needs torchrun with 2 or more ranks")
        run_tp(args, wl, shape)
    else:
        run_b200(args, wl, shape)


if __name__ == "__main__":
    main()
