"""The C-ABI library: it loads, exports every entry point the header
declares, and its host-only logic (config validation, arena sizing) holds.
No compute call is made, so these run without a GPU."""
import ctypes

import pytest

import decoder_only_b200 as lb
import oracle
from synth.workloads import PRESETS, TINY, LLAMA_7B, LLAMA_13B


def test_every_declared_symbol_is_exported():
    names = lb.header_symbols()
    assert len(names) >= 17
    for n in names:
        assert hasattr(lb.lib, n), n


def test_status_strings():
    for code in (0, -1, -2, -3, -4, -5):
        assert lb.lib.llama_status_str(code)


@pytest.mark.parametrize("name", sorted(PRESETS))
def test_arena_holds_every_parameter_and_the_kv_cache(name):
    shape = PRESETS[name]
    B, S = (32, 2304) if shape is LLAMA_13B else (4, 2176)
    cfg = lb.make_config(shape, B, S)
    nbytes = lb.model_bytes(cfg)
    esz = 2 if shape.dtype == "bf16" else 4
    gains = (2 * shape.n_layers + 1) * shape.d_model
    params = (oracle.count_params(shape) - gains) * esz + gains * 4
    kv = 2 * shape.n_layers * B * S * shape.d_model * esz
    assert nbytes >= params + kv
    assert nbytes < (params + kv) * 1.2 + (B * S) * shape.d_model * 40 + (1 << 30)


def test_hidden_size_rule_in_the_library_matches_the_oracle():
    # ffn_hidden = 0 asks the library for the rule; sizes differ iff the rule differs
    for d in (4096, 5120, 8192):
        s = LLAMA_7B.with_(d_model=d, n_heads=d // 128, ffn_hidden=oracle.llama_hidden(d), n_layers=1)
        explicit = lb.model_bytes(lb.make_config(s, 1, 64))
        rule = lb.model_bytes(lb.make_config(s.with_(ffn_hidden=0), 1, 64))
        assert explicit == rule


@pytest.mark.parametrize("bad", [
    dict(head_dim=100), dict(n_heads=3), dict(dtype="f16"), dict(ffn_hidden=100), dict(d_model=4096 + 32),
])
def test_invalid_configs_are_rejected(bad):
    s = LLAMA_7B.with_(**bad)
    cfg = lb.make_config(s, 4, 128)
    if bad.get("dtype") == "f16":
        cfg.dtype = 7
    n = ctypes.c_uint64()
    assert lb.lib.llama_model_bytes(ctypes.byref(cfg), ctypes.byref(n)) == -1


def test_bf16_batch_limit_and_tiny_fp32_accepted():
    assert lb.lib.llama_model_bytes(ctypes.byref(lb.make_config(LLAMA_7B, 33, 64)),
                                    ctypes.byref(ctypes.c_uint64())) == -1
    assert lb.model_bytes(lb.make_config(TINY, 1, 32)) > 0
