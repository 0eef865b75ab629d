"""Build and call ``brute.c`` (the C triple-loop oracle) through ctypes.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "brute.c")
_LIB = os.path.join(_HERE, "_brute.so")
_handle = None


def build_brute(force: bool = False) -> str:
    """Compile brute.c into oracle/_brute.so with gcc (plain -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.run(["gcc", "-O2", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _lib():
    global _handle
    if _handle is None:
        _handle = ctypes.CDLL(build_brute())
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int32)
        _handle.brute_attention.argtypes = [dp, dp, dp, dp, dp] + [ctypes.c_int] * 5 + [ctypes.c_double]
        _handle.brute_attention.restype = None
        _handle.brute_paged_decode.argtypes = [dp, dp, dp, ip, ip, ctypes.c_int, dp, dp] + [ctypes.c_int] * 4 + [ctypes.c_double]
        _handle.brute_paged_decode.restype = None
    return _handle


def _dp(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def brute_attention(Q, K, V, causal: bool, scale: float):
    """[B, H, N, d] float arrays -> (O, LSE) in float64 via brute.c."""
    Q, K, V = (np.ascontiguousarray(x, dtype=np.float64) for x in (Q, K, V))
    B, H, N, d = Q.shape
    O = np.zeros_like(Q)
    LSE = np.zeros((B, H, N))
    _lib().brute_attention(_dp(Q), _dp(K), _dp(V), _dp(O), _dp(LSE), B, H, N, d, int(causal), float(scale))
    return O, LSE


def brute_paged_decode(q, k_cache, v_cache, block_table, seq_lens, block_size: int, scale: float):
    """Paged decode via brute.c; block-table entries must be valid."""
    q, kc, vc = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k_cache, v_cache))
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    sl = np.ascontiguousarray(seq_lens, dtype=np.int32)
    S, H, d = q.shape
    O = np.zeros_like(q)
    LSE = np.zeros((S, H))
    ip = ctypes.POINTER(ctypes.c_int32)
    _lib().brute_paged_decode(_dp(q), _dp(kc), _dp(vc), bt.ctypes.data_as(ip), sl.ctypes.data_as(ip),
                              int(block_size), _dp(O), _dp(LSE), S, H, d, bt.shape[1], float(scale))
    return O, LSE
