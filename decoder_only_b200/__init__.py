"""Python binding of libllama_b200.so: argument marshalling only.

Every step of the forward pass runs in the library's CUDA kernels; PyTorch
supplies device memory (one arena tensor per model) and the current stream.
Importing this package without the built library raises ImportError: there
is no other implementation to fall back to.
"""
from __future__ import annotations

import ctypes
import os
import re
import traceback

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libllama_b200.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "llama_b200.h")

F32, BF16 = 0, 1
STATUS = {0: "ok", -1: "invalid argument", -2: "arena or workspace too small", -3: "CUDA error",
          -4: "bounded device wait expired", -5: "call out of order"}


class LlamaError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        super().__init__(f"{what}: {STATUS.get(code, code)} ({code})")
        self.code = code


class LlamaConfig(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int32), ("d_model", ctypes.c_int32), ("n_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("ffn_hidden", ctypes.c_int32), ("vocab", ctypes.c_int32),
                ("norm_eps", ctypes.c_float), ("rope_theta", ctypes.c_float), ("dtype", ctypes.c_int32),
                ("max_batch", ctypes.c_int32), ("max_seq", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("bias", ctypes.c_int32), ("tp_size", ctypes.c_int32), ("tp_rank", ctypes.c_int32),
                ("kv_pages", ctypes.c_int32)]


# int (*)(float* d_buf, uint64_t count, void* stream, void* ctx): the exchange of a shard
ALLREDUCE_FN = ctypes.CFUNCTYPE(ctypes.c_int, ctypes.c_void_p, ctypes.c_uint64, ctypes.c_void_p, ctypes.c_void_p)


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python decoder_only_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, U64, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint64, ctypes.c_float
    sig = {
        "llama_model_bytes": [P, P],
        "llama_init_weights": [P, ctypes.c_uint32, P, U64, P, P],
        "llama_prefill": [P, P, I, I, P, P],
        "llama_prefill_ragged": [P, P, I, I, P, P, P],
        "llama_positions": [P, P, I],
        "llama_prefill_trunk": [P, P, I, I, P, P],
        "llama_decode_step": [P, P, P, P, P],
        "llama_generate": [P, P, I, P, P],
        "llama_position": [P],
        "llama_model_tensor": [P, ctypes.c_char_p, I, P, P],
        "llama_last_error": [P],
        "llama_free": [P],
        "llama_status_str": [ctypes.c_int],
        "llama_op_rmsnorm": [I, P, P, P, I, I, F, P],
        "llama_op_gemm": [I, P, P, P, I, I, I, I, P],
        "llama_op_attention_prefill": [I, P, P, P, P, I, I, I, I, I, P],
        "llama_op_attention_decode": [I, P, P, P, P, I, I, I, I, I, P, U64, P],
        "llama_op_attention_decode_work_bytes": [I, I, I, I],
        "llama_op_attention_decode_noalloc": [I, P, P, P, P, I, I, I, I, I, P],
        "llama_op_argmax": [P, I, I, P, P],
        "llama_op_last_error": [],
        "llama_set_allreduce": [P, ALLREDUCE_FN, P, I],
        "llama_tp_shard": [P, P],
        "llama_set_pages": [P, P, I, I, P],
        "llama_rewind": [P, I, P],
        "llama_complete": [P, P, I, I, P, I, P, P],
        "llama_kernel_launches": [],
        "llama_step_timeline": [P, P, ctypes.c_int64, P, P],
        "llama_debug_gemm_timeout": [P],
        "llama_profile_enable": [I],
        "llama_profile_reset": [],
        "llama_profile_count": [],
        "llama_profile_entry": [I, P, P, P, P, P, P],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    lib.llama_free.restype = None
    lib.llama_profile_reset.restype = None
    lib.llama_kernel_launches.restype = ctypes.c_int64
    lib.llama_status_str.restype = ctypes.c_char_p
    lib.llama_op_attention_decode_work_bytes.restype = U64
    return lib


lib = _load()


def header_symbols() -> list[str]:
    """Names of the entry points include/llama_b200.h declares."""
    with open(HEADER_PATH) as f:
        return re.findall(r"^LLAMA_API\s+[\w\s\*]+?\b(llama_\w+)\s*\(", f.read(), flags=re.M)


def _check(rc: int, what: str):
    if rc != 0:
        raise LlamaError(rc, what)


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t: torch.Tensor | None):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def make_config(shape, max_batch: int, max_seq: int, tp=None, kv_pages: int = 0) -> LlamaConfig:
    """`shape`: any object with n_layers, d_model, n_heads, head_dim,
    ffn_hidden, vocab, dtype ('bf16' | 'f32'), norm_eps, rope_theta.
    `tp`: (rank, size) of a tensor-parallel shard, or None.  `kv_pages`:
    pages of 128 positions in a paged KV cache (0: contiguous)."""
    rank, size = tp if tp is not None else (0, 0)
    return LlamaConfig(shape.n_layers, shape.d_model, shape.n_heads, shape.head_dim, shape.ffn_hidden,
                       shape.vocab, shape.norm_eps, shape.rope_theta, BF16 if shape.dtype == "bf16" else F32,
                       max_batch, max_seq, int(getattr(shape, "n_kv_heads", 0) or 0),
                       int(bool(getattr(shape, "bias", False))), size, rank, kv_pages)


def tp_shard(shape, rank: int, size: int) -> dict:
    """The slices shard `rank` of `size` holds (llama_tp_shard)."""
    cfg = make_config(shape, 1, 1, (rank, size))
    out = (ctypes.c_int32 * 6)()
    _check(lib.llama_tp_shard(ctypes.byref(cfg), ctypes.cast(out, ctypes.c_void_p)), "llama_tp_shard")
    return dict(head0=out[0], heads=out[1], kv_head0=out[2], kv_heads=out[3], hidden0=out[4], hidden=out[5])


def allreduce_callback(resolve, reduce):
    """The C exchange (llama_allreduce_fn) around two Python callables:
    resolve(ptr, count) -> the float32 tensor of `count` elements at `ptr`;
    reduce(buf, stream) queues the sum over the shards of `buf` in place on
    `stream` (a torch stream, or None for host tensors).  Exceptions are
    printed and reported to the library as a failed exchange."""
    streams = {}

    def cb(ptr, count, stream, ctx):
        try:
            buf = resolve(ptr or 0, int(count))
            st = None
            if stream:
                st = streams.get(stream)
                if st is None:
                    st = streams[stream] = torch.cuda.ExternalStream(stream)
            reduce(buf, st)
            return 0
        except Exception:
            traceback.print_exc()
            return 1

    return ALLREDUCE_FN(cb)


def dist_allreduce(group=None):
    """reduce(buf, stream) for allreduce_callback / Model.set_allreduce: one
    torch.distributed sum all-reduce (NCCL between GPUs) queued on `stream`."""
    import torch.distributed as dist

    def reduce(buf, stream):
        if stream is None:
            dist.all_reduce(buf, group=group)
        else:
            with torch.cuda.stream(stream):
                dist.all_reduce(buf, group=group)

    return reduce


def model_bytes(cfg: LlamaConfig) -> int:
    n = ctypes.c_uint64()
    _check(lib.llama_model_bytes(ctypes.byref(cfg), ctypes.byref(n)), "llama_model_bytes")
    return n.value


class Model:
    """One model in one device arena.  Weights are generated on the device."""

    def __init__(self, shape, max_batch: int, max_seq: int, seed: int = 0, tp=None, kv_pages: int = 0):
        self.shape = shape
        self.cfg = make_config(shape, max_batch, max_seq, tp, kv_pages)
        nbytes = model_bytes(self.cfg)
        self.arena = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        h = ctypes.c_void_p()
        _check(lib.llama_init_weights(ctypes.byref(self.cfg), seed, _ptr(self.arena), nbytes, _stream(),
                                      ctypes.byref(h)), "llama_init_weights")
        self.h = h
        self.wdtype = torch.bfloat16 if shape.dtype == "bf16" else torch.float32

    def close(self):
        if self.h:
            lib.llama_free(self.h)
            self.h = None

    def set_pages(self, table):
        """Page table of a paged KV cache (llama_set_pages): table[b][p] is the
        pool page of sequence b's positions 128 p .. 128 p + 127."""
        rows = [list(map(int, r)) for r in table]
        B, n = len(rows), len(rows[0])
        flat = (ctypes.c_int32 * (B * n))(*[v for r in rows for v in r])
        _check(lib.llama_set_pages(self.h, ctypes.cast(flat, ctypes.c_void_p), B, n, _stream()), "llama_set_pages")

    def set_allreduce(self, reduce, chunks: int = 4):
        """Installs the exchange of a tensor-parallel shard (llama_set_allreduce):
        reduce(buf, stream) sums `buf`, a float32 view of trunk rows in this
        model's arena, over the shards in place on `stream`."""
        arena = self.arena

        def resolve(ptr, count):
            off = ptr - arena.data_ptr()
            return arena[off:off + 4 * count].view(torch.float32)

        self._allreduce_cb = allreduce_callback(resolve, reduce)   # kept alive with the model
        _check(lib.llama_set_allreduce(self.h, self._allreduce_cb, None, chunks), "llama_set_allreduce")

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def position(self) -> int:
        return lib.llama_position(self.h)

    def prefill(self, tokens: torch.Tensor, logits: bool = True, out: torch.Tensor | None = None,
                lens=None):
        """tokens int32 [B, S] on the device -> logits fp32 [B, S, V] (or None).
        With ``lens`` (B ints) the batch is ragged: sequence b is its first
        lens[b] tokens (llama_prefill_ragged)."""
        B, S = tokens.shape
        tokens = tokens.contiguous()
        if logits and out is None:
            out = torch.empty(B, S, self.cfg.vocab, dtype=torch.float32, device="cuda")
        if lens is None:
            _check(lib.llama_prefill(self.h, _ptr(tokens), B, S, _ptr(out if logits else None), _stream()),
                   "llama_prefill")
        else:
            h_lens = (ctypes.c_int32 * B)(*[int(x) for x in lens])
            _check(lib.llama_prefill_ragged(self.h, _ptr(tokens), B, S, ctypes.cast(h_lens, ctypes.c_void_p),
                                            _ptr(out if logits else None), _stream()), "llama_prefill_ragged")
        return out if logits else None

    def positions(self):
        """Each sequence's decode position (host ints)."""
        cap = max(int(self.cfg.max_batch), 1)
        buf = (ctypes.c_int32 * cap)()
        n = lib.llama_positions(self.h, ctypes.cast(buf, ctypes.c_void_p), cap)
        _check(min(n, 0), "llama_positions")
        return [buf[i] for i in range(n)]

    def complete(self, tokens_host: torch.Tensor, n_steps: int, logits: torch.Tensor | None = None,
                 out_host: torch.Tensor | None = None) -> torch.Tensor:
        """Host int32 [B, S] prompt -> host int32 [n_steps, B] greedy tokens
        (llama_complete; pass pinned tensors for asynchronous copies)."""
        B, S = tokens_host.shape
        if out_host is None:
            out_host = torch.empty(n_steps, B, dtype=torch.int32, pin_memory=True)
        _check(lib.llama_complete(self.h, _ptr(tokens_host.contiguous()), B, S, _ptr(logits), n_steps,
                                  _ptr(out_host), _stream()), "llama_complete")
        return out_host

    def rewind(self, position: int):
        _check(lib.llama_rewind(self.h, position, _stream()), "llama_rewind")

    def prefill_trunk(self, x: torch.Tensor, out: torch.Tensor | None = None):
        """x fp32 [B, S, d] -> trunk after the blocks, fp32 [B, S, d]."""
        B, S, _ = x.shape
        x = x.contiguous()
        y = torch.empty_like(x) if out is None else out
        _check(lib.llama_prefill_trunk(self.h, _ptr(x), B, S, _ptr(y), _stream()), "llama_prefill_trunk")
        return y

    def decode_step(self, tokens: torch.Tensor, logits: bool = True):
        B = tokens.shape[0]
        nxt = torch.empty(B, dtype=torch.int32, device="cuda")
        lg = torch.empty(B, self.cfg.vocab, dtype=torch.float32, device="cuda") if logits else None
        _check(lib.llama_decode_step(self.h, _ptr(tokens.contiguous()), _ptr(nxt), _ptr(lg), _stream()),
               "llama_decode_step")
        return nxt, lg

    def generate(self, first: torch.Tensor | None, n_steps: int, out: torch.Tensor | None = None,
                 batch: int | None = None):
        """n_steps greedy tokens [n_steps, B]; first=None continues from the
        prefill's own greedy choice."""
        B = first.shape[0] if first is not None else batch
        out = torch.empty(n_steps, B, dtype=torch.int32, device="cuda") if out is None else out
        f = None if first is None else first.contiguous()
        _check(lib.llama_generate(self.h, _ptr(f), n_steps, _ptr(out), _stream()), "llama_generate")
        return out

    def tensor(self, name: str, layer: int = 0, dtype=None, shape=None) -> torch.Tensor:
        """A view of an internal buffer (see llama_model_tensor)."""
        p, n = ctypes.c_void_p(), ctypes.c_uint64()
        _check(lib.llama_model_tensor(self.h, name.encode(), layer, ctypes.byref(p), ctypes.byref(n)),
               "llama_model_tensor")
        off = p.value - self.arena.data_ptr()
        t = self.arena[off:off + n.value]
        if dtype is not None:
            t = t.view(dtype)
        if shape is not None:
            t = t[: int(torch.Size(shape).numel())].view(shape)
        return t

    def step_timeline(self):
        """[ctas, phases, 2] ns stamps of the last decode step run while
        profiling was enabled (bf16 models)."""
        import numpy as np
        c, p = ctypes.c_int32(), ctypes.c_int32()
        _check(lib.llama_step_timeline(self.h, None, 0, ctypes.byref(c), ctypes.byref(p)), "llama_step_timeline")
        out = np.zeros((c.value, p.value, 2), dtype=np.uint64)
        _check(lib.llama_step_timeline(self.h, ctypes.c_void_p(out.ctypes.data), out.size, None, None),
               "llama_step_timeline")
        return out

    def last_error(self) -> int:
        return lib.llama_last_error(self.h)


# ----------------------------------------------------------------- instrumentation

def kernel_launches() -> int:
    return int(lib.llama_kernel_launches())


def profile_enable(on: bool = True):
    lib.llama_profile_enable(1 if on else 0)


def profile_reset():
    lib.llama_profile_reset()


def profile_read() -> dict:
    """{region: dict(ms, launches, calls, bytes, flops)} (synchronises)."""
    out = {}
    for i in range(lib.llama_profile_count()):
        name = ctypes.c_char_p()
        ms, by, fl = ctypes.c_double(), ctypes.c_double(), ctypes.c_double()
        la, ca = ctypes.c_int64(), ctypes.c_int64()
        _check(lib.llama_profile_entry(i, ctypes.byref(name), ctypes.byref(ms), ctypes.byref(la), ctypes.byref(ca),
                                       ctypes.byref(by), ctypes.byref(fl)), "llama_profile_entry")
        out[name.value.decode()] = dict(ms=ms.value, launches=la.value, calls=ca.value, bytes=by.value,
                                        flops=fl.value)
    return out


# ----------------------------------------------------------------- single ops

def rmsnorm(x: torch.Tensor, g: torch.Tensor, eps: float, out_dtype=torch.bfloat16) -> torch.Tensor:
    rows, d = x.shape
    y = torch.empty(rows, d, dtype=out_dtype, device=x.device)
    _check(lib.llama_op_rmsnorm(_dt(y), _ptr(x.contiguous()), _ptr(g.contiguous()), _ptr(y), rows, d, eps,
                                _stream()), "llama_op_rmsnorm")
    return y


def gemm(A: torch.Tensor, W: torch.Tensor, C: torch.Tensor | None = None, accumulate: bool = False):
    """C (+)= A W^T, A [M, K], W [N, K] (same dtype), C fp32 [M, N]."""
    M, K = A.shape
    N = W.shape[0]
    if C is None:
        C = torch.empty(M, N, dtype=torch.float32, device=A.device)
    _check(lib.llama_op_gemm(_dt(A), _ptr(A.contiguous()), _ptr(W.contiguous()), _ptr(C), M, N, K,
                             1 if accumulate else 0, _stream()), "llama_op_gemm")
    return C


def attention_prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor) -> torch.Tensor:
    """q [B, H, S, hd]; k, v [B, H, kv_stride, hd] -> o [B*S, H*hd]."""
    B, H, S, hd = q.shape
    kv_stride = k.shape[2]
    o = torch.empty(B * S, H * hd, dtype=q.dtype, device=q.device)
    _check(lib.llama_op_attention_prefill(_dt(q), _ptr(q.contiguous()), _ptr(k.contiguous()), _ptr(v.contiguous()),
                                          _ptr(o), B, H, S, hd, kv_stride, _stream()), "llama_op_attention_prefill")
    return o


def attention_decode(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, length: int,
                     work: torch.Tensor | None = None) -> torch.Tensor:
    """q [B, H*hd]; k, v [B, H, kv_stride, hd]; keys 0..length-1 -> o [B, H*hd]."""
    B, H, kv_stride, hd = k.shape
    nbytes = lib.llama_op_attention_decode_work_bytes(B, H, length, hd)
    if work is None:
        work = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    o = torch.empty(B, H * hd, dtype=q.dtype, device=q.device)
    _check(lib.llama_op_attention_decode(_dt(q), _ptr(q.contiguous()), _ptr(k.contiguous()), _ptr(v.contiguous()),
                                         _ptr(o), B, H, length, hd, kv_stride, _ptr(work), work.numel(),
                                         _stream()), "llama_op_attention_decode")
    return o


def attention_decode_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, length: int) -> torch.Tensor:
    """attention_decode with the workspace in the library's fixed device
    array: no allocation by the library (see the header for the limit)."""
    B, H, kv_stride, hd = k.shape
    o = torch.empty(B, H * hd, dtype=q.dtype, device=q.device)
    _check(lib.llama_op_attention_decode_noalloc(_dt(q), _ptr(q.contiguous()), _ptr(k.contiguous()),
                                                 _ptr(v.contiguous()), _ptr(o), B, H, length, hd, kv_stride,
                                                 _stream()), "llama_op_attention_decode_noalloc")
    return o


def op_last_error() -> int:
    """Reads and clears the single ops' device error word (synchronises the
    current device): 0, or -4 when a bounded device wait expired."""
    return int(lib.llama_op_last_error())


def argmax(logits: torch.Tensor) -> torch.Tensor:
    rows, n = logits.shape
    out = torch.empty(rows, dtype=torch.int32, device=logits.device)
    _check(lib.llama_op_argmax(_ptr(logits.contiguous()), rows, n, _ptr(out), _stream()), "llama_op_argmax")
    return out
