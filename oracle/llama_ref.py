"""fp64 CPU oracle of the LLaMA pre-norm decoder forward pass.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or
links this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It
shares no code with the CUDA library; its inputs (random-init weights, token
ids) come from the seeded generator in ``synth``.

Plain, slow, obviously correct: every step is written out in fp64 NumPy in
the order the pages give it, with no blocking, fusion or reordering.

Sources (cited by page title and section):
  [PFD] "LLaMA: Open and Efficient Foundation Language Models",
        paperfordummies.in -- sections "The one formula",
        "RMSNorm: LayerNorm minus the mean", "Pre-norm: the norm goes on the
        branch, not the trunk", "SwiGLU: a gate in the FFN, paid for with a
        narrower hidden layer", "RoPE: rotate Q and K, leave V alone",
        "6.7B parameters, 1T tokens: the arithmetic", "The code".
  [NAR] "LLaMA: No Architecture Revolution, Yet It Became the Open-Model
        Foundation" -- sections "An Architecture Recipe Without an
        Invention Myth" (RMSNorm with gain g, SwiGLU, the RoPE relative-offset
        identity) and "GQA Was Not an Original LLaMA Feature" (KV cache).

Readings taken where the pages are silent:
  * RMSNorm carries the gain g of [NAR]; the gains are 1 in every workload.
  * RoPE acts per head (its d is the head dimension), on interleaved
    (even, odd) channel pairs, angle = position * base^(-2i/d_head).
  * Heads are contiguous blocks of d_head columns of Q, K, V.
  * The bias variant (the page's bias=True count): every linear layer adds a
    bias of its output width (Q, K, V before RoPE), and the two in-layer
    norms add a shift after the gain, z = x / rms(x) * g + beta; the final
    norm and the head have none (the count has none).  Biases and shifts are
    drawn N(0, 0.02^2) like the weights and kept in fp32.
  * Grouped keys and values ([NAR] "GQA Was Not an Original LLaMA
    Feature"; LLaMA itself has one K/V head per query head): with n_kv
    key/value heads, K and V have n_kv heads of d_head columns and query
    head h attends with key/value head floor(h / (H / n_kv)) -- contiguous
    groups of H / n_kv query heads.  n_kv = H is the original model.
  * Attention scale 1/sqrt(d_head); the causal mask keeps key j <= query t.
  * Prefill returns logits for every position; decoding is greedy with the
    lowest token id winning ties.
  * Activations stay fp64 here by default; only the weights are rounded to
    the storage type the workload names.  With storage="bf16" the oracle
    also rounds (nearest-even, from fp64) every value a bf16 workload stores
    in bf16: the normalised inputs of the projections, Q, K and V (the KV
    cache is bf16), the attention output and the SwiGLU activation.  That
    variant exists to measure how far bf16 storage alone moves the result:
    the GPU must be no less accurate than it (see tests/test_oracle_pins.py
    for why a fixed 2e-2 bound cannot hold at depth with a bf16 KV cache).

Pinning: every function below is pinned by tests in tests/test_oracle_pins.py
against values the pages print, closed forms, invariants, brute force or a
library routine.  The pages print no forward-pass output, so the end-to-end
logits are pinned only through those pinned steps and the invariants
(causality, prefix truncation, decode == prefill row, pre-norm identity).
"""
from __future__ import annotations

import math

import numpy as np

import synth


# ----------------------------------------------------------------------------
# scalar and row primitives
# ----------------------------------------------------------------------------

def rms_norm(x: np.ndarray, g: np.ndarray | None = None, eps: float = 1e-6) -> np.ndarray:
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps), times gain g.

    [PFD] "RMSNorm: LayerNorm minus the mean" (divide by the root-mean-square,
    no mean subtraction, no shift); [NAR] "An Architecture Recipe Without an
    Invention Myth" gives the gain g.
    """
    x = np.asarray(x, dtype=np.float64)
    mean_sq = np.mean(np.square(x), axis=-1, keepdims=True)
    y = x / np.sqrt(mean_sq + eps)
    if g is not None:
        y = y * np.asarray(g, dtype=np.float64)
    return y


def silu(u: np.ndarray) -> np.ndarray:
    """SiLU(u) = u * sigmoid(u) = u / (1 + e^-u).  [PFD] "The code" / SwiGLU."""
    u = np.asarray(u, dtype=np.float64)
    with np.errstate(over="ignore"):
        return u / (1.0 + np.exp(-u))


def llama_hidden(d_model: int, multiple_of: int = 256) -> int:
    """FFN hidden width: floor(2/3 * 4d), rounded up to a multiple of 256.

    [PFD] "SwiGLU: a gate in the FFN, paid for with a narrower hidden layer"
    (11008, not 10923, for d = 4096).
    """
    two_thirds = (8 * d_model) // 3
    return multiple_of * (-(-two_thirds // multiple_of))


def rope(x: np.ndarray, positions: np.ndarray, base: float = 10000.0) -> np.ndarray:
    """Rotary position embedding on the last axis (length d, even).

    Channel pair i = (x[2i], x[2i+1]) is rotated by angle p * base^(-2i/d),
    p the token's position.  Written as multiplication of the complex number
    x[2i] + 1j*x[2i+1] by exp(1j * angle), which is the same 2-D rotation.
    [PFD] "RoPE: rotate Q and K, leave V alone" and "The code"; [NAR]
    (R_m q)^T (R_n k) = q^T R_{n-m} k.

    x: (..., n, d) with positions (n,) broadcast over the leading axes.
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    assert d % 2 == 0
    i = np.arange(d // 2, dtype=np.float64)
    theta = base ** (-(2.0 * i) / d)                                   # (d/2,)
    angle = np.asarray(positions, dtype=np.float64)[:, None] * theta[None, :]  # (n, d/2)
    z = x[..., 0::2] + 1j * x[..., 1::2]
    z = z * np.exp(1j * angle)
    out = np.empty_like(x)
    out[..., 0::2] = z.real
    out[..., 1::2] = z.imag
    return out


def causal_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """Scaled dot-product attention with a causal mask, one head.

    q, k, v: (n, d_head).  Row t attends to keys j <= t:
    softmax_j(q_t . k_j / sqrt(d_head)) weighting v_j.  The softmax subtracts
    the row maximum before exponentiating.  [PFD] "LLaMA is a pull request
    against the 2017 transformer" (attention untouched, causal mask).
    """
    n, dh = q.shape
    scores = (q @ k.T) / math.sqrt(dh)
    future = np.triu(np.ones((n, n), dtype=bool), k=1)
    scores = np.where(future, -np.inf, scores)
    scores = scores - scores.max(axis=-1, keepdims=True)
    w = np.exp(scores)
    w = w / w.sum(axis=-1, keepdims=True)
    return w @ v


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest bf16 (ties to even), returned as fp64.

    Goes through fp32 with round-to-odd (truncate, then set the lowest bit
    when inexact), which makes the second rounding to bf16 exact."""
    x = np.asarray(x, dtype=np.float64)
    f = x.astype(np.float32)
    over = np.abs(f.astype(np.float64)) > np.abs(x)
    f = np.where(over, np.nextafter(f, np.float32(0)), f)
    inexact = f.astype(np.float64) != x
    b = f.view(np.uint32) | inexact.astype(np.uint32)
    b = ((b.astype(np.uint64) + 0x7FFF + ((b >> 16) & 1)) >> 16) << 16
    return b.astype(np.uint32).view(np.float32).astype(np.float64)


def _storer(storage, kv=False):
    """Rounding applied where a value is stored.  storage: None (exact),
    "bf16" (every bf16 storage point) or "bf16-kv" (only the KV cache)."""
    if storage is None or (storage == "bf16-kv" and not kv):
        return lambda x: x
    if storage in ("bf16", "bf16-kv"):
        return round_bf16
    raise ValueError(storage)


# ----------------------------------------------------------------------------
# weights
# ----------------------------------------------------------------------------

def weight_shapes(shape, bias: bool = False) -> dict:
    """Every parameter tensor of the model and its shape, in the (d_in, d_out)
    orientation in which the forward pass computes x @ W.

    [PFD] "6.7B parameters, 1T tokens: the arithmetic": four d x d attention
    matrices, three FFN matrices (3dh), two norms per layer, an embedding
    table, an untied output head and the final norm.  With ``bias`` every
    linear layer gets a bias of its output width and every in-layer norm a
    shift (the page's bias=True count).
    """
    d, h, V, L = shape.d_model, shape.ffn_hidden, shape.vocab, shape.n_layers
    kvd = _kv_heads(shape) * shape.head_dim
    out = {"embed": (V, d)}
    for l in range(L):
        out.update({
            f"{l}.wq": (d, d), f"{l}.wk": (d, kvd), f"{l}.wv": (d, kvd), f"{l}.wo": (d, d),
            f"{l}.wg": (d, h), f"{l}.wu": (d, h), f"{l}.wd": (h, d),
            f"{l}.g_attn": (d,), f"{l}.g_ffn": (d,),
        })
        if bias:
            out.update({
                f"{l}.bq": (d,), f"{l}.bk": (kvd,), f"{l}.bv": (kvd,), f"{l}.bo": (d,),
                f"{l}.bg": (h,), f"{l}.bu": (h,), f"{l}.bd": (d,),
                f"{l}.beta_attn": (d,), f"{l}.beta_ffn": (d,),
            })
    out["g_final"] = (d,)
    out["head"] = (d, V)
    return out


def count_params(shape, bias: bool = False) -> int:
    return int(sum(int(np.prod(s)) for s in weight_shapes(shape, bias).values()))


def _kv_heads(shape) -> int:
    """Key/value heads: n_kv_heads when the shape sets it, else one per query head."""
    return getattr(shape, "n_kv_heads", 0) or shape.n_heads


def _draw(seed, tensor_id, rows, cols, dtype):
    w = synth.normal_stored(seed, tensor_id, rows * cols, synth.WEIGHT_STD, dtype)
    return w.reshape(rows, cols)


def layer_weights(shape, layer: int, seed: int = 0) -> dict:
    """Random-init weights of one block (fp64 arrays holding values rounded to
    the storage dtype), N(0, 0.02^2), RMSNorm gains 1."""
    d, h = shape.d_model, shape.ffn_hidden
    kvd = _kv_heads(shape) * shape.head_dim
    dims = {"wq": (d, d), "wk": (d, kvd), "wv": (d, kvd), "wo": (d, d),
            "wg": (d, h), "wu": (d, h), "wd": (h, d)}
    W = {name: _draw(seed, synth.layer_tensor_id(layer, name), r, c, shape.dtype)
         for name, (r, c) in dims.items()}
    W["g_attn"] = np.ones(d)
    W["g_ffn"] = np.ones(d)
    if getattr(shape, "bias", False):
        vec = {"bq": d, "bk": kvd, "bv": kvd, "bo": d, "bg": h, "bu": h, "bd": d, "beta_attn": d, "beta_ffn": d}
        for name, n in vec.items():
            W[name] = _draw(seed, synth.layer_tensor_id(layer, name), 1, n, "f32")[0]
    return W


def _b(W, name):
    """A bias or shift of the bias variant; 0 in the original model."""
    return W.get(name, 0.0)


def embed_table(shape, seed: int = 0) -> np.ndarray:
    return _draw(seed, synth.EMBED, shape.vocab, shape.d_model, shape.dtype)


def head_matrix(shape, seed: int = 0) -> np.ndarray:
    return _draw(seed, synth.HEAD, shape.d_model, shape.vocab, shape.dtype)


# ----------------------------------------------------------------------------
# sublayers, block, model
# ----------------------------------------------------------------------------

def split_heads(m: np.ndarray, n_heads: int) -> np.ndarray:
    """(n, d) -> (H, n, d_head): head k is columns [k*d_head, (k+1)*d_head)."""
    n, d = m.shape
    return m.reshape(n, n_heads, d // n_heads).transpose(1, 0, 2)


def merge_heads(m: np.ndarray) -> np.ndarray:
    H, n, dh = m.shape
    return m.transpose(1, 0, 2).reshape(n, H * dh)


def attn_sublayer(z, W, positions, shape, kv_out=None, storage=None):
    """Q, K, V = z Wq, z Wk, z Wv; RoPE on Q and K (not V); causal attention
    per head; heads concatenated; times Wo.  [PFD] "RoPE: rotate Q and K,
    leave V alone" (where rope is applied)."""
    st, st_kv = _storer(storage), _storer(storage, kv=True)
    H, Hkv = shape.n_heads, _kv_heads(shape)
    G = H // Hkv                                   # query heads per key/value head
    q = split_heads(z @ W["wq"] + _b(W, "bq"), H)
    k = split_heads(z @ W["wk"] + _b(W, "bk"), Hkv)
    v = split_heads(z @ W["wv"] + _b(W, "bv"), Hkv)
    q = st(rope(q, positions, shape.rope_theta))
    k = st_kv(rope(k, positions, shape.rope_theta))
    v = st_kv(v)
    if kv_out is not None:
        kv_out.append((k, v))
    o = np.stack([causal_attention(q[hh], k[hh // G], v[hh // G]) for hh in range(H)])
    return st(merge_heads(o)) @ W["wo"] + _b(W, "bo")


def swiglu_ffn(z, W, storage=None):
    """(SiLU(z Wg) * (z Wu)) Wd, (n,d) -> (n,h) -> (n,d).  [PFD] SwiGLU;
    [NAR] SwiGLU(x) = SiLU(x W_g) (.) (x W_v)."""
    gate = silu(z @ W["wg"] + _b(W, "bg"))
    up = z @ W["wu"] + _b(W, "bu")
    return _storer(storage)(gate * up) @ W["wd"] + _b(W, "bd")


def pre_norm_block(x, W, positions, shape, kv_out=None, storage=None):
    """h = x + Attn(RMSNorm(x));  y = h + FFN(RMSNorm(h)).

    The norm sits on each branch; the trunk x is only ever added to.
    [PFD] "The one formula" and "Pre-norm: the norm goes on the branch, not
    the trunk"."""
    st = _storer(storage)
    z = rms_norm(x, W["g_attn"], shape.norm_eps) + _b(W, "beta_attn")
    h = x + attn_sublayer(st(z), W, positions, shape, kv_out, storage)
    z = rms_norm(h, W["g_ffn"], shape.norm_eps) + _b(W, "beta_ffn")
    y = h + swiglu_ffn(st(z), W, storage)
    return y


def prefill(shape, tokens: np.ndarray, seed: int = 0, weights=None, return_cache=False,
            return_trunk=False, storage=None):
    """Embedding -> L pre-norm blocks -> final RMSNorm -> untied head.

    tokens: (B, S) int.  Returns logits (B, S, V) for every position
    ([PFD] "The one formula": after block L, one final RMSNorm, then the
    output head, (n, 32000)).  No position signal is added at the bottom.
    ``weights``: optional callable layer -> dict (else drawn from ``synth``).
    With ``return_cache`` the per-layer (K after RoPE, V) of every sequence is
    returned as cache[l] = (K, V), each (B, n_kv, S, d_head).
    ``storage`` may be a tuple of storage modes: the forward pass then runs
    once per mode on the same weights (each layer drawn once) and a list of
    logits, one per mode, is returned.
    """
    multi = isinstance(storage, (tuple, list))
    modes = list(storage) if multi else [storage]
    tokens = np.asarray(tokens)
    B, S = tokens.shape
    E = embed_table(shape, seed)
    get_w = weights if weights is not None else (lambda l: layer_weights(shape, l, seed))
    xs = [[E[tokens[b]].copy() for b in range(B)] for _ in modes]
    positions = np.arange(S)
    cache = [] if return_cache else None
    for l in range(shape.n_layers):
        W = get_w(l)
        for mi, mode in enumerate(modes):
            kv = []
            for b in range(B):
                xs[mi][b] = pre_norm_block(xs[mi][b], W, positions, shape,
                                           kv if (return_cache and mi == 0) else None, mode)
            if return_cache and mi == 0:
                cache.append((np.stack([k for k, _ in kv]), np.stack([v for _, v in kv])))
        del W
    Wh = head_matrix(shape, seed)
    logits_all = []
    for mi, mode in enumerate(modes):
        trunk = np.stack(xs[mi])
        logits_all.append(_storer(mode)(rms_norm(trunk, np.ones(shape.d_model), shape.norm_eps)) @ Wh)
    if multi:
        return logits_all
    out = [logits_all[0]]
    if return_cache:
        out.append(cache)
    if return_trunk:
        out.append(np.stack(xs[0]))
    return out[0] if len(out) == 1 else tuple(out)


def decode_step(shape, cache: list, tokens: np.ndarray, seed: int = 0, weights=None):
    """One decoding step for a batch: each sequence's new token sits at
    position p = current cache length; its K, V are appended; it attends to
    positions 0..p.  Returns (logits (B, V), next tokens (B,), new cache).

    Written one token at a time, apart from the batched ``prefill`` path, so
    that decode == prefill-row is a check between two formulations.
    Greedy choice: argmax, lowest id on ties.  KV cache per [NAR] "GQA Was
    Not an Original LLaMA Feature" (keys and values of every previous token
    are cached).
    """
    tokens = np.asarray(tokens)
    B = tokens.shape[0]
    H, dh = shape.n_heads, shape.head_dim
    Hkv = _kv_heads(shape)
    G = H // Hkv
    E = embed_table(shape, seed)
    get_w = weights if weights is not None else (lambda l: layer_weights(shape, l, seed))
    p = cache[0][0].shape[2]
    x = E[tokens].copy()                                     # (B, d)
    new_cache = []
    for l in range(shape.n_layers):
        W = get_w(l)
        Kc, Vc = cache[l]
        z = rms_norm(x, W["g_attn"], shape.norm_eps) + _b(W, "beta_attn")
        q = (z @ W["wq"] + _b(W, "bq")).reshape(B, H, dh)
        k = (z @ W["wk"] + _b(W, "bk")).reshape(B, Hkv, dh)
        v = (z @ W["wv"] + _b(W, "bv")).reshape(B, Hkv, dh)
        pos = np.array([p])
        q = rope(q.reshape(B * H, 1, dh), pos, shape.rope_theta).reshape(B, H, dh)
        k = rope(k.reshape(B * Hkv, 1, dh), pos, shape.rope_theta).reshape(B, Hkv, dh)
        Kc = np.concatenate([Kc, k[:, :, None, :]], axis=2)
        Vc = np.concatenate([Vc, v[:, :, None, :]], axis=2)
        o = np.empty((B, H, dh))
        for b in range(B):
            for hh in range(H):
                s = Kc[b, hh // G] @ q[b, hh] / math.sqrt(dh)      # (p+1,)
                w = np.exp(s - s.max())
                o[b, hh] = (w / w.sum()) @ Vc[b, hh // G]
        x = x + o.reshape(B, H * dh) @ W["wo"] + _b(W, "bo")
        z = rms_norm(x, W["g_ffn"], shape.norm_eps) + _b(W, "beta_ffn")
        x = x + (silu(z @ W["wg"] + _b(W, "bg")) * (z @ W["wu"] + _b(W, "bu"))) @ W["wd"] + _b(W, "bd")
        new_cache.append((Kc, Vc))
        del W
    logits = rms_norm(x, np.ones(shape.d_model), shape.norm_eps) @ head_matrix(shape, seed)
    nxt = np.argmax(logits, axis=-1).astype(np.int32)      # first maximum = lowest id
    return logits, nxt, new_cache


def block_forward(shape, x: np.ndarray, layer: int = 0, seed: int = 0, weights=None, storage=None):
    """One pre-norm block on a given fp32 trunk x (S, d), positions 0..S-1."""
    W = weights if weights is not None else layer_weights(shape, layer, seed)
    return pre_norm_block(np.asarray(x, dtype=np.float64), W, np.arange(x.shape[0]), shape, storage=storage)
