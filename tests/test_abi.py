"""The C-ABI library: it loads, exports every entry point the header
declares, and its host-only logic (config validation, arena sizing) holds.
No compute call is made, so these run without a GPU."""
import ctypes

import pytest

import decoder_only_b200 as lb
import oracle
from synth.workloads import PRESETS, TINY, LLAMA_7B, LLAMA_13B, LLAMA_65B_SLICE


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


def _bytes(shape, B=4, S=128):
    n = ctypes.c_uint64()
    rc = lb.lib.llama_model_bytes(ctypes.byref(lb.make_config(shape, B, S)), ctypes.byref(n))
    return rc, n.value


def test_grouped_kv_heads_shrink_the_projection_and_the_cache_exactly():
    """n_kv key/value heads: W_k and W_v lose 2 d (H - n_kv) hd values per
    layer and the cache 2 L B S (H - n_kv) hd (the [NAR] KV-cache formula)."""
    s = LLAMA_7B.with_(n_layers=2)
    B, S = 4, 128
    rc, full = _bytes(s, B, S)
    rc8, gqa = _bytes(s.with_(n_kv_heads=8), B, S)
    assert rc == rc8 == 0
    hd, H, L, d = s.head_dim, s.n_heads, s.n_layers, s.d_model
    saved = 2 * (L * 2 * d * (H - 8) * hd + 2 * L * B * S * (H - 8) * hd)   # bf16 bytes
    # beyond that only the decode step's split-K partials of the narrower QKV
    # projection change (fp32, [rows][slots][B]), plus 256-byte alignment
    qkv_partials = 4 * 3 * d * 8 * B
    assert saved - 256 * 64 <= full - gqa <= saved + qkv_partials


@pytest.mark.parametrize("n_kv", [3, -1, 64])
def test_grouped_kv_heads_must_divide_the_query_heads(n_kv):
    assert _bytes(LLAMA_7B.with_(n_layers=1, n_kv_heads=n_kv))[0] == -1


def test_bias_variant_adds_its_vectors():
    """Per layer: b_qkv, b_o, b_gu, b_d, two shifts, and the decode step's two
    folded biases, fp32 (the page's +1,622,016 values for 7B plus the folds)."""
    s = LLAMA_7B.with_(n_layers=2)
    rc0, plain = _bytes(s)
    rc1, biased = _bytes(s.with_(bias=True))
    assert rc0 == rc1 == 0
    d, h, L = s.d_model, s.ffn_hidden, s.n_layers
    per_layer = (3 * d + d + 2 * h + d + 2 * d) + (3 * d + 2 * h)
    assert biased - plain >= 4 * L * per_layer
    assert biased - plain < 4 * L * per_layer + 256 * 16 * L + 4096


def test_code_hash_ignores_comments_not_code(tmp_path):
    import bench
    a = tmp_path / "a.cu"
    a.write_text('int f(int x) {  // twice\n  return 2 * x; /* doubled */ }\nconst char* s = "// kept";\n')
    b = tmp_path / "b.cu"
    b.write_text('int f(int x) {\n  return 2 * x;\n}\nconst char* s = "// kept";  // other words\n')
    c = tmp_path / "c.cu"
    c.write_text('int f(int x) {\n  return 3 * x;\n}\nconst char* s = "// kept";\n')
    assert bench.code_hash(str(a)) == bench.code_hash(str(b))
    assert bench.code_hash(str(a)) != bench.code_hash(str(c))


# ------------------------------------------------------------------ tensor parallel (host logic)

@pytest.mark.parametrize("shape,T", [(LLAMA_7B, 2), (LLAMA_13B, 2), (LLAMA_13B, 4), (LLAMA_7B.with_(n_kv_heads=8), 2),
                                     (LLAMA_65B_SLICE, 4)])
def test_tp_shards_partition_heads_and_hidden_units(shape, T):
    """Every query head, key/value head and FFN hidden unit belongs to
    exactly one shard, in contiguous rank-ordered slices."""
    if True:
        sh = [lb.tp_shard(shape, r, T) for r in range(T)]
        for key0, key, total in (("head0", "heads", shape.n_heads), ("kv_head0", "kv_heads", shape.kv_heads),
                                 ("hidden0", "hidden", shape.ffn_hidden)):
            assert [s[key0] for s in sh] == [r * total // T for r in range(T)]
            assert all(s[key] == total // T for s in sh)


def test_tp_shard_holds_its_slice_of_the_weights_and_cache():
    """A shard's arena is the unsharded one minus (T - 1) / T of the sharded
    weights (Q, K, V, O, gate, up, down) and of the KV cache."""
    s = LLAMA_7B.with_(n_layers=2)
    B, S = 4, 128
    full = lb.model_bytes(lb.make_config(s, B, S))
    half = lb.model_bytes(lb.make_config(s, B, S, tp=(1, 2)))
    d, h, L = s.d_model, s.ffn_hidden, s.n_layers
    sharded = 2 * L * (4 * d * d + 3 * d * h) + 2 * 2 * L * B * S * d          # bf16 bytes
    act = B * S * (2 * d + h) * 2                                              # q, attention output, SwiGLU act
    saved = full - half
    # beyond that: the decode step's split-K partial regions, sized by the widths the model holds
    assert sharded // 2 <= saved <= sharded // 2 + act // 2 + (1 << 20)


@pytest.mark.parametrize("tp", [(0, 3), (2, 2), (-1, 2), (1, 1), (0, 256), (0, 4)])
def test_tp_configs_that_do_not_divide_are_rejected(tp):
    # 7B: 32 heads, 11008 = 86 blocks of 128 hidden units: 4 shards would split a block
    n = ctypes.c_uint64()
    cfg = lb.make_config(LLAMA_7B.with_(n_layers=1), 4, 128, tp=tp)
    assert lb.lib.llama_model_bytes(ctypes.byref(cfg), ctypes.byref(n)) == -1


def test_tp_exchange_is_rejected_on_an_unsharded_model_handle():
    assert lb.lib.llama_set_allreduce(None, lb.ALLREDUCE_FN(lambda *a: 0), None, 4) == -1


# ------------------------------------------------------------------ paged KV cache (host logic)

def test_paged_cache_arena_holds_the_pool_instead_of_the_slabs():
    s = LLAMA_7B.with_(n_layers=2)
    B, S = 4, 1000
    contiguous = lb.model_bytes(lb.make_config(s, B, S))
    paged = lb.model_bytes(lb.make_config(s, B, S, kv_pages=11))
    kv = 2 * s.n_layers * B * S * s.d_model * 2
    pool = 2 * s.n_layers * 11 * 128 * s.d_model * 2
    table = B * 8 * 4
    assert contiguous - kv == pytest.approx(paged - pool - table, abs=256 * 4)


def test_paged_cache_needs_bf16():
    n = ctypes.c_uint64()
    assert lb.lib.llama_model_bytes(ctypes.byref(lb.make_config(TINY, 1, 32, kv_pages=2)), ctypes.byref(n)) == -1
    assert lb.lib.llama_model_bytes(ctypes.byref(lb.make_config(LLAMA_7B, 1, 32, kv_pages=-1)),
                                    ctypes.byref(n)) == -1


def test_every_entry_point_cites_its_passage_or_says_it_has_none():
    """Each declaration in the header comes after a comment that cites the page
    passage defining its operation ([PFD], [NAR], [KN] tags) or states that
    there is none (bookkeeping, inspection, instrumentation, failure detection)."""
    import re
    from pathlib import Path
    src = (Path(__file__).resolve().parent.parent / "include" / "llama_b200.h").read_text()
    missing = []
    for m in re.finditer(r"^LLAMA_API[^(]*?(\w+)\s*\(", src, re.M):
        before = src[:m.start()]
        comment = before[before.rfind("/*"):before.rfind("*/")]
        if not re.search(r"\[(PFD|NAR|KN)\]|No passage", comment):
            missing.append(m.group(1))
    assert not missing, missing
