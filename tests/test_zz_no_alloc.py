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


def _inputs(B, H, kv_stride, hd, tid):
    q = synth.normal(11, tid, B * H * hd).reshape(B, H * hd)
    k = synth.normal(11, tid + 1, B * H * kv_stride * hd).reshape(B, H, kv_stride, hd)
    v = synth.normal(11, tid + 2, B * H * kv_stride * hd).reshape(B, H, kv_stride, hd)
    return [torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).cuda() for x in (q, k, v)]


@pytest.mark.gpu
def test_noalloc_matches_the_workspace_entry_point_on_consecutive_calls():
    # two calls in a row with different shapes: nothing of the first leaks into the second
    for (B, H, length, hd), tid in (((4, 32, 2049, 128), 100), ((3, 5, 300, 64), 200)):
        q, k, v = _inputs(B, H, length + 3, hd, tid)
        ref = lb.attention_decode(q, k, v, length)
        got = lb.attention_decode_noalloc(q, k, v, length)
        torch.cuda.synchronize()
        r = ref.float().cpu().numpy()
        g = got.float().cpu().numpy()
        rms = np.sqrt(np.mean(r ** 2))
        assert np.all(np.abs(g - r) <= 2.0 ** -8 * np.abs(r) + 2e-3 * rms)


def test_noalloc_rejects_workspace_beyond_the_limit_before_any_cuda_call():
    # host-side validation only: the pointers are never dereferenced
    fake = ctypes.c_void_p(256)
    rc = lb.lib.llama_op_attention_decode_noalloc(1, fake, fake, fake, fake, 64, 64, 2304, 128, 2304, None)
    assert rc == -2
    rc = lb.lib.llama_op_attention_decode_noalloc(1, fake, fake, fake, fake, 4, 32, 10, 100, 16, None)
    assert rc == -1
