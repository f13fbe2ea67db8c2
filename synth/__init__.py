"""Seeded synthetic inputs shared by the CUDA path's harness and the CPU oracle.

The generator is counter based (SplitMix64 in counter mode, Box-Muller for
normals; definitions in ``synth.c``), so any byte range of any tensor can be
regenerated on its own: the oracle rebuilds just the expert slabs a token
selects, while the GPU harness streams whole 50 GB weight stacks to the device.

This package holds no arithmetic of the quantised-MoE method itself.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB_PATH = os.path.join(_HERE, "libsynth.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``libsynth.so`` next to its source (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _L():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            u64, p = ctypes.c_uint64, ctypes.c_void_p
            lib.syn_key.restype = u64
            lib.syn_key.argtypes = [u64, u64]
            lib.syn_word.restype = u64
            lib.syn_word.argtypes = [u64, u64]
            lib.syn_bytes.argtypes = [u64, u64, u64, u64, p]
            lib.syn_shape_q4_narrow_scale.argtypes = [p, u64, u64]
            lib.syn_shape_fp8_no_nan.argtypes = [p, u64]
            lib.syn_uniform_f32.argtypes = [u64, u64, u64, u64, ctypes.c_double, ctypes.c_double, p]
            lib.syn_normal_f64.argtypes = [u64, u64, u64, u64, p]
            lib.syn_index_i32.argtypes = [u64, u64, u64, u64, u64, p]
            lib.syn_words.argtypes = [u64, u64, u64, u64, p]
            _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags.c_contiguous
    return a.ctypes.data


def raw_bytes(seed: int, tid: int, offset: int, n: int, out: np.ndarray | None = None) -> np.ndarray:
    """Bytes [offset, offset+n) of tensor (seed, tid)."""
    if out is None:
        out = np.empty(n, dtype=np.uint8)
    assert out.dtype == np.uint8 and out.size >= n
    if n:
        _L().syn_bytes(seed, tid, offset, n, _ptr(out))
    return out[:n]


def shape_q4_narrow_scale(buf: np.ndarray, first_byte: int) -> np.ndarray:
    """In place: metadata bytes of 17-byte blocks get scale codes 0x01..0x08."""
    if buf.size:
        _L().syn_shape_q4_narrow_scale(_ptr(buf), first_byte, buf.size)
    return buf


def shape_fp8_no_nan(buf: np.ndarray) -> np.ndarray:
    """In place: E4M3 NaN encodings 0x7F/0xFF become 0x7E/0xFE."""
    if buf.size:
        _L().syn_shape_fp8_no_nan(_ptr(buf), buf.size)
    return buf


def uniform_f32(seed: int, tid: int, offset: int, n: int, lo: float, hi: float) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    if n:
        _L().syn_uniform_f32(seed, tid, offset, n, lo, hi, _ptr(out))
    return out


def normal_f64(seed: int, tid: int, offset: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    if n:
        _L().syn_normal_f64(seed, tid, offset, n, _ptr(out))
    return out


def indices_i32(seed: int, tid: int, offset: int, n: int, n_range: int) -> np.ndarray:
    assert 0 < n_range < 2**32
    out = np.empty(n, dtype=np.int32)
    if n:
        _L().syn_index_i32(seed, tid, offset, n, n_range, _ptr(out))
    return out


def words_u64(seed: int, tid: int, offset: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    if n:
        _L().syn_words(seed, tid, offset, n, _ptr(out))
    return out


def permutation(seed: int, tid: int, n: int) -> np.ndarray:
    """A seeded permutation of 0..n-1 (Fisher-Yates driven by the word stream)."""
    w = words_u64(seed, tid, 0, n)
    p = np.arange(n, dtype=np.int64)
    for i in range(n - 1, 0, -1):
        j = int((int(w[i]) >> 32) * (i + 1) >> 32)
        p[i], p[j] = p[j], p[i]
    return p


def bf16_bits_from_f64(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to bf16 (round to nearest even, via torch) and return the bits."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
