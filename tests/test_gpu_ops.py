"""GPU parity of the single kernels, through the C ABI, against the fp64
oracle (or fp64 NumPy for a plain matrix product) on the same inputs."""
import numpy as np
import pytest
import torch

import decoder_only_b200 as lb
import oracle
import synth

pytestmark = pytest.mark.gpu


def _normal_bf16(tid, shape, scale=1.0):
    n = int(np.prod(shape))
    bits = synth.normal_bf16_bits(7, tid, n, scale).reshape(shape)
    t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
    return t, synth.bf16_bits_to_f64(bits.reshape(-1)).reshape(shape)


def _rms(a):
    return float(np.sqrt(np.mean(np.square(a))))


def _acc_bound(K):
    """Relative bound of an fp32 tensor-core accumulation over K: the bf16
    products are exact, each of the K/16 MMA steps adds one fp32 rounding of
    the running sum (not necessarily to nearest, so the errors can add up in
    one direction): (K/16) * 2^-22, and no less than 2e-5."""
    return max(2e-5, (K / 16) * 2.0 ** -22)


# ------------------------------------------------------------------ RMSNorm

@pytest.mark.parametrize("rows,d", [(1, 128), (33, 128), (7, 4096), (130, 5120), (3, 8192)])
@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_rmsnorm(rows, d, out):
    x = synth.normal(7, 100 + d, rows * d).reshape(rows, d) * 3.0
    g = 1.0 + 0.1 * synth.normal(7, 200 + d, d)
    xt = torch.from_numpy(x.astype(np.float32)).cuda()
    gt = torch.from_numpy(g.astype(np.float32)).cuda()
    y = lb.rmsnorm(xt, gt, 1e-6, torch.float32 if out == "f32" else torch.bfloat16)
    ref = oracle.rms_norm(x.astype(np.float32).astype(np.float64), g.astype(np.float32), 1e-6)
    got = y.float().cpu().numpy().astype(np.float64)
    if out == "f32":
        assert np.max(np.abs(got - ref)) <= 2e-6 * _rms(ref)
    else:   # one rounding to bf16 (relative 2^-9) on top of fp32 arithmetic
        assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6 * _rms(ref))


def test_rmsnorm_zero_rows_eps():
    x = torch.zeros(4, 128, device="cuda")
    g = torch.ones(128, device="cuda")
    assert torch.all(lb.rmsnorm(x, g, 1e-5, torch.float32) == 0)


# ------------------------------------------------------------------ tcgen05 GEMM

GEMM_SHAPES = [
    (1, 256, 64), (128, 256, 64), (127, 272, 128), (300, 512, 4096), (256, 4096, 11008),
    (2048, 12288, 4096), (8192, 32000, 4096),
]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_gemm_tc_matches_fp64(M, N, K):
    A, a64 = _normal_bf16(11, (M, K))
    W, w64 = _normal_bf16(12, (N, K), 0.02)
    C = lb.gemm(A, W)
    torch.cuda.synchronize()
    rows = np.arange(M) if M <= 512 else np.unique(np.concatenate(
        [np.arange(0, 130), np.random.default_rng(0).integers(0, M, 200), np.arange(M - 130, M)]))
    ref = a64[rows] @ w64.T
    got = C[torch.from_numpy(rows).cuda()].cpu().numpy().astype(np.float64)
    err = np.max(np.abs(got - ref))
    assert err <= _acc_bound(K) * _rms(ref), (err, _rms(ref))


def test_gemm_tc_accumulate():
    M, N, K = 200, 512, 1024
    A, a64 = _normal_bf16(13, (M, K))
    W, w64 = _normal_bf16(14, (N, K), 0.02)
    C0 = torch.from_numpy(synth.normal(7, 15, M * N).reshape(M, N).astype(np.float32)).cuda()
    c0 = C0.double().cpu().numpy()
    lb.gemm(A, W, C0, accumulate=True)
    ref = c0 + a64 @ w64.T
    assert np.max(np.abs(C0.cpu().numpy() - ref)) <= _acc_bound(K) * _rms(ref)


def test_gemm_tc_rejects_unsupported_shapes():
    A = torch.zeros(4, 100, dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(64, 100, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lb.LlamaError):
        lb.gemm(A, W)


def test_gemm_fp32_simt():
    M, N, K = 70, 130, 96
    a = synth.normal(7, 16, M * K).reshape(M, K)
    w = synth.normal(7, 17, N * K).reshape(N, K) * 0.02
    C = lb.gemm(torch.from_numpy(a.astype(np.float32)).cuda(), torch.from_numpy(w.astype(np.float32)).cuda())
    ref = a.astype(np.float32).astype(np.float64) @ w.astype(np.float32).astype(np.float64).T
    assert np.max(np.abs(C.cpu().numpy() - ref)) <= 1e-5 * _rms(ref)


# ------------------------------------------------------------------ attention

def _qkv(B, H, S, hd, kv_stride, dtype):
    n = B * H * S * hd
    qs = synth.normal(7, 21, n).reshape(B, H, S, hd)
    ks = synth.normal(7, 22, B * H * kv_stride * hd).reshape(B, H, kv_stride, hd)
    vs = synth.normal(7, 23, B * H * kv_stride * hd).reshape(B, H, kv_stride, hd)
    # inputs are rounded to the storage type on the host; the reference
    # reads the host copies, never the device
    host = [torch.from_numpy(x.astype(np.float32)).to(dtype) for x in (qs, ks, vs)]
    ref = [t.double().numpy() for t in host]
    dev = [t.cuda() for t in host]
    return (*dev, *ref)


@pytest.mark.parametrize("B,H,S,hd,dtype", [
    (1, 2, 1, 32, torch.float32), (1, 4, 37, 32, torch.float32), (2, 3, 130, 64, torch.float32),
    (1, 2, 200, 128, torch.bfloat16), (2, 2, 64, 64, torch.bfloat16),
    # a single key; one valid row in the last query tile; a ragged tail at head_dim 64
    (1, 2, 1, 128, torch.bfloat16), (1, 3, 129, 128, torch.bfloat16), (2, 2, 257, 64, torch.bfloat16),
])
def test_attention_prefill(B, H, S, hd, dtype):
    kv_stride = S + 5
    q, k, v, q64, k64, v64 = _qkv(B, H, S, hd, kv_stride, dtype)
    o = lb.attention_prefill(q, k, v).float().cpu().numpy().reshape(B, S, H, hd)
    for b in range(B):
        for h in range(H):
            ref = oracle.causal_attention(q64[b, h], k64[b, h, :S], v64[b, h, :S])
            got = o[b, :, h, :]
            if dtype == torch.float32:
                assert np.max(np.abs(got - ref)) <= 1e-5 * max(_rms(ref), 1e-3)
            else:
                assert np.all(np.abs(got - ref) <= _bf16_attn_bound(ref, v64[b, h, :S]))


def _bf16_attn_bound(ref, v):
    """Per-element bound of the bf16 attention: the probabilities are rounded
    to bf16 before P.V (relative 2^-9 each), which moves a weighted average
    by at most 2^-9 * sum_j w_j |v_j - o| <= 2^-8 max_j |v_j|; the output is
    rounded once more (2^-9 |o|); fp32 accumulation adds far less."""
    return 2.0 ** -8 * np.abs(ref) + 2.0 ** -8 * np.max(np.abs(v), axis=0)[None, :] + 1e-6


def test_attention_prefill_full_length_sampled_heads():
    B, H, S, hd = 1, 32, 2048, 128
    q, k, v, q64, k64, v64 = _qkv(B, H, S, hd, S, torch.bfloat16)
    o = lb.attention_prefill(q, k, v).float().cpu().numpy().reshape(B, S, H, hd)
    for h in (0, 17, 31):
        ref = oracle.causal_attention(q64[0, h], k64[0, h], v64[0, h])
        assert np.all(np.abs(o[0, :, h] - ref) <= _bf16_attn_bound(ref, v64[0, h]))
        # and far inside it on average
        assert _rms(o[0, :, h] - ref) <= 2e-3 * _rms(ref) + 2.0 ** -12


@pytest.mark.parametrize("B,H,length,hd,dtype", [
    (1, 1, 1, 128, torch.bfloat16), (4, 32, 2049, 128, torch.bfloat16), (3, 5, 300, 64, torch.bfloat16),
    (2, 4, 33, 32, torch.float32), (1, 4, 513, 128, torch.float32),
])
def test_attention_decode(B, H, length, hd, dtype):
    kv_stride = length + 7
    q, k, v, q64, k64, v64 = _qkv(B, H, 1, hd, kv_stride, dtype)
    o = lb.attention_decode(q.reshape(B, H * hd), k, v, length).float().cpu().numpy().reshape(B, H, hd)
    for b in range(B):
        for h in range(H):
            # the query as the last row of a causal window over keys 0..length-1
            qrow = np.zeros((length, hd))
            qrow[-1] = q64[b, h, 0]
            ref = oracle.causal_attention(qrow, k64[b, h, :length], v64[b, h, :length])[-1]
            if dtype == torch.float32:
                assert np.max(np.abs(o[b, h] - ref)) <= 1e-5 * max(_rms(ref), 1e-3)
            else:
                assert np.all(np.abs(o[b, h] - ref) <= 2.0 ** -8 * np.abs(ref) + 2e-3 * _rms(ref))


def test_argmax_lowest_index_on_ties():
    x = torch.zeros(3, 1000, device="cuda")
    x[0, 5] = 1.0
    x[1, 7] = 2.0
    x[1, 900] = 2.0
    # row 2: all equal -> 0
    assert lb.argmax(x).tolist() == [5, 7, 0]
    y = torch.randn(16, 32000, device="cuda")
    assert torch.equal(lb.argmax(y).long(), torch.argmax(y, dim=-1))


def test_bounded_wait_expires_and_the_context_survives():
    """Failure detection: a GEMM whose activation tile is never requested
    must give up after its bounded wait, report LLAMA_ERR_TIMEOUT, and leave
    the context usable (a normal GEMM right after is correct)."""
    assert lb.lib.llama_debug_gemm_timeout(lb._stream()) == -4
    A, a64 = _normal_bf16(31, (256, 512))
    W, w64 = _normal_bf16(32, (256, 512), 0.02)
    C = lb.gemm(A, W)
    ref = a64 @ w64.T
    assert np.max(np.abs(C.cpu().numpy() - ref)) <= _acc_bound(512) * _rms(ref)
