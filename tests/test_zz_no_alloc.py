"""The decode-attention entry point that allocates nothing.

Callers that cannot allocate device memory when they run a decode step
(pre-planned serving runtimes, graph-capture code that must not allocate,
embedders without a device allocator) use
llama_op_attention_decode_noalloc, whose workspace is a fixed array in the
library's own device memory.  Its results must match the workspace-taking
entry point, call after call.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import decoder_only_b200 as lb
import synth

LIMIT = 8 << 20   # bytes of the library's fixed workspace array


def _inputs(B, H, kv_stride, hd, tid, dtype):
    q = synth.normal(11, tid, B * H * hd).reshape(B, H * hd)
    k = synth.normal(11, tid + 1, B * H * kv_stride * hd).reshape(B, H, kv_stride, hd)
    v = synth.normal(11, tid + 2, B * H * kv_stride * hd).reshape(B, H, kv_stride, hd)
    return [torch.from_numpy(x.astype(np.float32)).to(dtype).cuda() for x in (q, k, v)]


def _close(got, ref, dtype):
    r = ref.float().cpu().numpy()
    g = got.float().cpu().numpy()
    rms = np.sqrt(np.mean(r ** 2))
    rel = 2.0 ** -8 if dtype == torch.bfloat16 else 2.0 ** -20
    assert np.all(np.abs(g - r) <= rel * np.abs(r) + 2e-3 * rms)


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,cases", [
    (torch.bfloat16, [((4, 32, 2049, 128), 100), ((3, 5, 300, 64), 200)]),
    (torch.float32, [((2, 4, 700, 32), 300), ((5, 3, 129, 128), 400)]),
    (torch.float32, [((1, 7, 1, 64), 500), ((2, 8, 4097, 32), 600)]),
])
def test_noalloc_matches_the_workspace_entry_point_on_consecutive_calls(dtype, cases):
    # two calls in a row with different shapes: nothing of the first leaks into the second
    for (B, H, length, hd), tid in cases:
        q, k, v = _inputs(B, H, length + 3, hd, tid, dtype)
        ref = lb.attention_decode(q, k, v, length)
        got = lb.attention_decode_noalloc(q, k, v, length)
        torch.cuda.synchronize()
        _close(got, ref, dtype)
    assert lb.op_last_error() == 0


@pytest.mark.gpu
def test_noalloc_runs_at_the_limit_and_rejects_one_chunk_more():
    # B * H = 64 pairs of head_dim 128: 4 * 64 * 130 bytes per 128-key chunk;
    # 252 chunks (32256 keys) fill 8386816 of the 8388608 bytes, 253 do not fit
    B, H, hd, length = 2, 32, 128, 252 * 128
    assert lb.lib.llama_op_attention_decode_work_bytes(B, H, length, hd) <= LIMIT
    assert lb.lib.llama_op_attention_decode_work_bytes(B, H, length + 1, hd) > LIMIT
    g = torch.Generator(device="cuda").manual_seed(7)
    q = torch.randn(B, H * hd, device="cuda", generator=g).to(torch.bfloat16)
    k = torch.randn(B, H, length + 1, hd, device="cuda", generator=g).to(torch.bfloat16)
    v = torch.randn(B, H, length + 1, hd, device="cuda", generator=g).to(torch.bfloat16)
    for _ in range(2):
        ref = lb.attention_decode(q, k, v, length)
        got = lb.attention_decode_noalloc(q, k, v, length)
        torch.cuda.synchronize()
        _close(got, ref, torch.bfloat16)
    with pytest.raises(lb.LlamaError) as e:
        lb.attention_decode_noalloc(q, k, v, length + 1)
    assert e.value.code == -2
    assert lb.op_last_error() == 0


def test_noalloc_rejects_workspace_beyond_the_limit_before_any_cuda_call():
    # host-side validation only: the pointers are never dereferenced
    fake = ctypes.c_void_p(256)
    rc = lb.lib.llama_op_attention_decode_noalloc(1, fake, fake, fake, fake, 64, 64, 2304, 128, 2304, None)
    assert rc == -2
    rc = lb.lib.llama_op_attention_decode_noalloc(1, fake, fake, fake, fake, 2, 32, 252 * 128 + 1, 128,
                                                  252 * 128 + 1, None)
    assert rc == -2
    rc = lb.lib.llama_op_attention_decode_noalloc(1, fake, fake, fake, fake, 4, 32, 10, 100, 16, None)
    assert rc == -1
