"""Seeded synthetic inputs, shared by the oracle, the tests and the bench.

This module holds none of the attention arithmetic. It maps
(seed, tensor id, element index) to a bf16 bit pattern: a counter-based
SplitMix64 stream, Box-Muller normals in float64, a per-config factor, then a
single round-to-nearest-even to bfloat16. The C source (``synth.c``) states the
exact recipe; this file only builds and calls it.

Tensor ids: Q=0, K=1, V=2, x=3, Wq=4, Wk=5, Wv=6, Wo=7, dO (upstream gradient)=8.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

TENSOR_IDS = {"q": 0, "k": 1, "v": 2, "x": 3, "wq": 4, "wk": 5, "wv": 6, "wo": 7, "do": 8}

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``libsynth.so`` next to its source (gcc + OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            i64, u64, u32, dbl, vp = (ctypes.c_int64, ctypes.c_uint64, ctypes.c_uint32,
                                      ctypes.c_double, ctypes.c_void_p)
            lib.synth_fill_bf16.argtypes = [vp, i64, i64, u64, u32, dbl]
            lib.synth_fill_bf16.restype = None
            lib.synth_fill_f64.argtypes = [vp, i64, i64, u64, u32, dbl]
            lib.synth_fill_f64.restype = None
            lib.synth_double_to_bf16.argtypes = [dbl]
            lib.synth_double_to_bf16.restype = ctypes.c_uint16
            lib.synth_sample_indices.argtypes = [vp, i64, i64, u64]
            lib.synth_sample_indices.restype = None
            lib.synth_mix64.argtypes = [u64]
            lib.synth_mix64.restype = u64
            _lib = lib
    return _lib


def _tid(tensor) -> int:
    return TENSOR_IDS[tensor] if isinstance(tensor, str) else int(tensor)


def fill_bf16_into(ptr: int, n: int, seed: int, tensor, factor: float = 1.0, offset: int = 0) -> None:
    """Write n bf16 values (as uint16 bits) to host memory at ``ptr``."""
    _load().synth_fill_bf16(ctypes.c_void_p(ptr), n, offset, seed, _tid(tensor), factor)


def bf16_bits(shape, seed: int, tensor, factor: float = 1.0) -> np.ndarray:
    """Return a uint16 array of bf16 bit patterns with the given shape."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    if n:
        fill_bf16_into(out.ctypes.data, n, seed, tensor, factor)
    return out.reshape(shape)


def normal_f64(shape, seed: int, tensor, factor: float = 1.0) -> np.ndarray:
    """The same stream before bf16 rounding (float64)."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float64)
    if n:
        _load().synth_fill_f64(ctypes.c_void_p(out.ctypes.data), n, 0, seed, _tid(tensor), factor)
    return out.reshape(shape)


def double_to_bf16_bits(x: float) -> int:
    return int(_load().synth_double_to_bf16(float(x)))


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def sample_rows(n: int, limit: int, seed: int, must_include=()) -> np.ndarray:
    """Seeded, sorted, de-duplicated indices in [0, limit), plus ``must_include``."""
    n = int(min(n, limit))
    raw = np.empty(max(n, 1), dtype=np.int64)
    _load().synth_sample_indices(ctypes.c_void_p(raw.ctypes.data), n, limit, seed)
    idx = set(int(i) for i in raw[:n])
    idx.update(int(i) for i in must_include if 0 <= int(i) < limit)
    # top up if duplicates removed too many
    k = n
    while len(idx) < n:
        extra = np.empty(1, dtype=np.int64)
        _load().synth_sample_indices(ctypes.c_void_p(extra.ctypes.data), 1, limit, seed + 7919 * (k + 1))
        idx.add(int(extra[0]))
        k += 1
    return np.array(sorted(idx), dtype=np.int64)


def mix64(x: int) -> int:
    return int(_load().synth_mix64(x))
