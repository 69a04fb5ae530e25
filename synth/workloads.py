"""Workload shapes the benchmarks and parity tests run on.

Plain data: model widths, depths, batch and sequence sizes, seeds.  The FFN
hidden sizes are stated here as the numbers the workloads name (they equal
the 2/3 * 4d rule rounded up to a multiple of 256; the oracle's own rule is
tested against them).
"""
from __future__ import annotations

from dataclasses import dataclass, asdict, replace


@dataclass(frozen=True)
class ModelShape:
    name: str
    n_layers: int
    d_model: int
    n_heads: int
    head_dim: int
    ffn_hidden: int
    vocab: int
    dtype: str = "bf16"          # storage type of weights and GEMM operands: 'bf16' or 'f32'
    norm_eps: float = 1e-6
    rope_theta: float = 10000.0
    n_kv_heads: int = 0          # key/value heads (GQA / MQA); 0: one per query head
    bias: bool = False           # the bias variant: linear biases and norm shifts

    @property
    def kv_heads(self) -> int:
        return self.n_kv_heads or self.n_heads

    def as_dict(self):
        return asdict(self)

    def with_(self, **kw) -> "ModelShape":
        return replace(self, **kw)


SEED = 0

# Tiny LLaMA, fp32 end to end; prefill of 1 x 32 tokens.
TINY = ModelShape("tiny-fp32", 2, 128, 4, 32, 512, 1000, dtype="f32")
# One 7B-shaped block (no embedding/head used); 1 x 2048 trunk N(0,1).
BLOCK_7B = ModelShape("llama-7b-block", 1, 4096, 32, 128, 11008, 32000)
# Full 7B shape: 32 layers.  Prefill 4 x 2048, then 128 greedy decode steps.
LLAMA_7B = ModelShape("llama-7b", 32, 4096, 32, 128, 11008, 32000)
# 13B shape: 40 layers.  Decode-heavy: batch 32, 2048-token prompts, 256 steps.
LLAMA_13B = ModelShape("llama-13b", 40, 5120, 40, 128, 13824, 32000)
# 33B shape: 60 layers, d 6656 = 52 heads of 128, hidden 17920.
LLAMA_33B = ModelShape("llama-33b", 60, 6656, 52, 128, 17920, 32000)
# 65B widths, 16 of 80 layers.  Prefill 8 x 2048 (+ S in {512,1024,2048} x B in {1,8}).
LLAMA_65B_SLICE = ModelShape("llama-65b-slice16", 16, 8192, 64, 128, 22016, 32000)

PRESETS = {m.name: m for m in (TINY, BLOCK_7B, LLAMA_7B, LLAMA_13B, LLAMA_65B_SLICE)}

# Workload runs (model, batch, prompt length, decode steps)
RUNS = {
    "tiny": dict(model=TINY, batch=1, seq=32, decode_steps=0),
    "7b-block": dict(model=BLOCK_7B, batch=1, seq=2048, decode_steps=0),
    "7b": dict(model=LLAMA_7B, batch=4, seq=2048, decode_steps=128),
    "13b-decode": dict(model=LLAMA_13B, batch=32, seq=2048, decode_steps=256),
    "65b-slice": dict(model=LLAMA_65B_SLICE, batch=8, seq=2048, decode_steps=0),
}
