"""Seeded synthetic inputs: random-init weights, token ids, trunk activations.

This module holds none of the decoder's arithmetic.  It defines the inputs
the workloads run on -- weights N(0, 0.02^2) with RMSNorm gains 1, token ids
uniform over the vocabulary, an N(0, 1) fp32 trunk for the single-block
workload -- through one counter-based generator (Philox4x32-10 + Box-Muller,
specified in ``philox.c``).  The oracle and the tests draw their inputs here;
the CUDA library has its own device implementation of the same published
generator, and the tests check the two agree.

Tensor ids (the generator key's second word):
    EMBED = 1, HEAD = 2, TOKENS = 3, TRUNK = 4,
    layer l, matrix m  ->  16 + 8*l + m  with m = wq 0, wk 1, wv 2, wo 3,
                                              wg 4, wu 5, wd 6;
    layer l, bias k    ->  2^20 + 16*l + k with k = bq 0, bk 1, bv 2, bo 3,
                           bg 4, bu 5, bd 6, beta_attn 7, beta_ffn 8
                           (the bias variant: linear biases, norm shifts).
Element e of a matrix is its row-major index in the (d_in, d_out)
orientation in which the forward pass multiplies ``x @ W``; the embedding
table is (V, d) row-major.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "philox.c")
_LIB = os.path.join(_HERE, "_synth.so")

EMBED = 1
HEAD = 2
TOKENS = 3
TRUNK = 4
_MATRIX = {"wq": 0, "wk": 1, "wv": 2, "wo": 3, "wg": 4, "wu": 5, "wd": 6}
WEIGHT_STD = 0.02


_BIAS = {"bq": 0, "bk": 1, "bv": 2, "bo": 3, "bg": 4, "bu": 5, "bd": 6, "beta_attn": 7, "beta_ffn": 8}
BIAS_BASE = 1 << 20


def layer_tensor_id(layer: int, name: str) -> int:
    if name in _BIAS:
        return BIAS_BASE + 16 * layer + _BIAS[name]
    return 16 + 8 * layer + _MATRIX[name]


def build(force: bool = False) -> str:
    """Compile the generator with gcc (OpenMP) into synth/_synth.so."""
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        u32, u64, dbl = ctypes.c_uint32, ctypes.c_uint64, ctypes.c_double
        p = ctypes.c_void_p
        lib.synth_philox4x32_10.argtypes = [p, p, p]
        lib.synth_normal_f64.argtypes = [u32, u32, u64, u64, dbl, p]
        lib.synth_normal_stored_f64.argtypes = [u32, u32, u64, u64, dbl, ctypes.c_int, p]
        lib.synth_normal_bf16.argtypes = [u32, u32, u64, u64, dbl, p]
        lib.synth_normal_f32.argtypes = [u32, u32, u64, u64, dbl, p]
        lib.synth_tokens.argtypes = [u32, u32, u64, u64, u32, p]
        lib.synth_f64_to_bf16.argtypes = [dbl]
        lib.synth_f64_to_bf16.restype = ctypes.c_uint16
        _lib = lib
    return _lib


def philox4x32_10(counter, key) -> np.ndarray:
    c = np.ascontiguousarray(counter, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    out = np.empty(4, dtype=np.uint32)
    _load().synth_philox4x32_10(c.ctypes.data, k.ctypes.data, out.ctypes.data)
    return out


def normal(seed: int, tensor_id: int, count: int, scale: float = 1.0, first: int = 0) -> np.ndarray:
    """scale * z_e for e in [first, first+count), fp64, not rounded."""
    out = np.empty(count, dtype=np.float64)
    _load().synth_normal_f64(seed, tensor_id, first, count, scale, out.ctypes.data)
    return out


def normal_stored(seed: int, tensor_id: int, count: int, scale: float, dtype: str,
                  first: int = 0) -> np.ndarray:
    """The same draw rounded (nearest-even, from fp64) into ``dtype``
    ('bf16' or 'f32'); returned as exactly-representable fp64 values."""
    out = np.empty(count, dtype=np.float64)
    _load().synth_normal_stored_f64(seed, tensor_id, first, count, scale,
                                    1 if dtype == "bf16" else 0, out.ctypes.data)
    return out


def normal_bf16_bits(seed: int, tensor_id: int, count: int, scale: float, first: int = 0) -> np.ndarray:
    out = np.empty(count, dtype=np.uint16)
    _load().synth_normal_bf16(seed, tensor_id, first, count, scale, out.ctypes.data)
    return out


def normal_f32(seed: int, tensor_id: int, count: int, scale: float, first: int = 0) -> np.ndarray:
    out = np.empty(count, dtype=np.float32)
    _load().synth_normal_f32(seed, tensor_id, first, count, scale, out.ctypes.data)
    return out


def tokens(seed: int, count: int, vocab: int, tensor_id: int = TOKENS, first: int = 0) -> np.ndarray:
    """Token ids uniform over [0, vocab): (r0 * vocab) >> 32, integer exact."""
    out = np.empty(count, dtype=np.int32)
    _load().synth_tokens(seed, tensor_id, first, count, vocab, out.ctypes.data)
    return out


def f64_to_bf16_bits(x: float) -> int:
    return int(_load().synth_f64_to_bf16(float(x)))


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)
