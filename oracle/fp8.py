"""fp64 CPU oracle for the FP8 (e4m3) quantisation of Q and K.

TEST INFRASTRUCTURE ONLY (see the package docstring): used by ``tests/``
and the CPU legs of ``bench.py``, never by the library.

Source: [技术详解] "一文掌握大模型推理加速：FlashAttention与PagedAttention技术详解"
§二 "FlashAttention-3改进" (hardware-accelerated low-precision GEMM: the
forward pass targets FP8 tensor cores, and block quantisation plus
incoherent processing limit the accuracy lost in the FP8 conversion) and
"性能提升" (the FP8 version has 2.6x lower numerical error than baseline FP8
attention).

Readings (the pages name the two techniques and nothing more):

* FP8 is e4m3 in its finite-only form: 1 sign, 4 exponent bits (bias 7),
  3 mantissa bits; normal values (1 + m/8) 2^(e-7), e = 1..15 with
  (e, m) = (15, 7) reserved, so the largest value is 448; subnormals
  (m/8) 2^-6.  Conversion rounds to nearest, ties to an even mantissa, and
  saturates beyond 448 (no infinities).
* Block quantisation: one scale per block of 128 consecutive rows of one
  head (the tile height of the attention kernel), chosen from the block's
  absolute maximum so that it maps to 448.
* Incoherent processing: each row (length d, a power of two) is multiplied
  by D H, D a diagonal of random signs drawn once (an input here) and H the
  Sylvester Hadamard matrix; (Q D H)(K D H)^T = d Q K^T, so the 1/sqrt(d)
  that makes the rotation orthogonal is folded into the stored scale and
  the dequantised operands give Q K^T unchanged.  It spreads an outlier
  coordinate over all d coordinates before the block maximum is taken.

The exact arithmetic of one block (both sides take the code decision in
fp32, the precision of the kernel):

    y      = x D H               (rows; without rotation y = x)
    amax   = max |y|             (fp32)
    r      = fp32(448 / amax)    (amax = 0: r = 1; overflow: largest fp32)
    code   = e4m3(fp32(y * r))   (round to nearest even, saturating)
    scale  = fp32(amax / (448 * sqrt(d)))  with rotation, fp32(amax / 448)
             without (amax = 0: 1)

and the dequantised value of a code is code * scale.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E4M3_MIN_SUBNORMAL = 2.0 ** -9


def _e4m3_grid() -> np.ndarray:
    """All non-negative finite e4m3 values, ascending (codes 0x00 .. 0x7e)."""
    vals = [m / 8.0 * 2.0 ** -6 for m in range(8)]  # subnormals and zero
    for e in range(1, 16):
        for m in range(8):
            if e == 15 and m == 7:
                continue  # NaN
            vals.append((1.0 + m / 8.0) * 2.0 ** (e - 7))
    return np.array(vals, dtype=np.float64)


E4M3_GRID = _e4m3_grid()


def e4m3_round(x) -> np.ndarray:
    """Round to the nearest e4m3 value, ties to the even code (even mantissa),
    saturating at +-448.  Returns float64 values on the e4m3 grid; NaN stays
    NaN."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    g = E4M3_GRID
    hi = np.clip(np.searchsorted(g, a, side="left"), 0, len(g) - 1)  # first grid value >= a
    lo = np.clip(hi - 1, 0, len(g) - 1)
    dlo = a - g[lo]
    dhi = g[hi] - a
    # index parity = code parity = mantissa parity (codes are consecutive)
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    out = np.where(pick_hi, g[hi], g[lo])
    out = np.where(a >= g[-1], g[-1], out)  # saturate
    out = np.where(a == 0, 0.0, out)
    out = np.copysign(out, x)
    return np.where(np.isnan(x), np.nan, out)


def e4m3_code(v) -> np.ndarray:
    """The 8-bit encoding of values already on the e4m3 grid."""
    v = np.asarray(v, dtype=np.float64)
    idx = np.searchsorted(E4M3_GRID, np.abs(v))
    if not np.all(E4M3_GRID[np.clip(idx, 0, len(E4M3_GRID) - 1)] == np.abs(v)):
        raise ValueError("value not on the e4m3 grid")
    return (idx | np.where(np.signbit(v), 0x80, 0)).astype(np.uint8)


def e4m3_decode(codes) -> np.ndarray:
    """Value of 8-bit e4m3 codes (0x7f / 0xff are NaN)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    mag = c & 0x7F
    out = np.where(mag == 0x7F, np.nan, E4M3_GRID[np.minimum(mag, len(E4M3_GRID) - 1)])
    return np.where(c & 0x80, -out, out)


def hadamard(d: int) -> np.ndarray:
    """Sylvester Hadamard matrix of order d (a power of two), entries +-1."""
    if d < 1 or d & (d - 1):
        raise ValueError("d must be a power of two")
    H = np.ones((1, 1))
    while H.shape[0] < d:
        H = np.block([[H, H], [H, -H]])
    return H


def rotate(x, signs) -> np.ndarray:
    """Incoherent processing of rows: x D H (unnormalised), fp64."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    return (x * np.asarray(signs, dtype=np.float64)) @ hadamard(d)


def quantize_blocks(x, block_rows: int = 128, signs=None):
    """Block-quantise rows of x [..., N, d] (fp32 values, e.g. bf16 inputs
    upcast) to e4m3.

    ``signs`` (d values of +-1) selects incoherent processing: the rows are
    rotated here, in fp64 (:func:`rotate`), and rounded to fp32 before the
    code decision.  Returns (codes as float64 values on the e4m3 grid,
    scales float32 [..., nblk]).
    """
    x = np.asarray(x, dtype=np.float32)
    *lead, N, d = x.shape
    if signs is not None:
        y = rotate(x, signs).astype(np.float32)
    else:
        y = x
    nblk = -(-N // block_rows)
    codes = np.zeros(y.shape, dtype=np.float64)
    scales = np.zeros(tuple(lead) + (nblk,), dtype=np.float32)
    for b in range(nblk):
        r0, r1 = b * block_rows, min(N, (b + 1) * block_rows)
        blk = y[..., r0:r1, :]
        amax = np.abs(blk).max(axis=(-2, -1)).astype(np.float32)
        with np.errstate(divide="ignore", over="ignore"):
            r = np.float32(448.0) / amax
        r = np.where(amax == 0, np.float32(1.0), r)
        r = np.where(np.isinf(r), np.finfo(np.float32).max, r).astype(np.float32)
        prod = (blk * r[..., None, None]).astype(np.float32)
        codes[..., r0:r1, :] = e4m3_round(prod)
        denom = 448.0 * np.sqrt(d) if signs is not None else 448.0
        sc = np.where(amax == 0, 1.0, amax.astype(np.float64) / denom).astype(np.float32)
        scales[..., b] = sc
    return codes, scales


def dequantize_blocks(codes, scales, block_rows: int = 128) -> np.ndarray:
    """codes * scale per block, fp64."""
    codes = np.asarray(codes, dtype=np.float64)
    N = codes.shape[-2]
    s = np.repeat(np.asarray(scales, dtype=np.float64), block_rows, axis=-1)[..., :N]
    return codes * s[..., None]
