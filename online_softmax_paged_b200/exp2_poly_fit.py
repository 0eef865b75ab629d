"""Fit of the cubic that the prefill softmax evaluates on the FMA pipe.

The bf16 prefill kernel exponentiates part of each score row with a
polynomial instead of the special-function unit: 2^x = 2^n * 2^f with
n = round(x) and f = x - n in [-1/2, 1/2], and 2^f ~ c0 + c1 f + c2 f^2 +
c3 f^3 (Horner, fp32 FMAs).  This module derives c0..c3.

Method: a weighted least-squares fit on Chebyshev nodes of [-1/2, 1/2] with
weights 1 / 2^f (relative error), refined by Lawson's iteration (the weights
are multiplied by the pointwise error and renormalised each round), which
drives the weighted least-squares solution towards the minimax (equioscillating)
one for relative error.  The coefficients are then rounded to fp32.

``python -m online_softmax_paged_b200.exp2_poly_fit`` prints them as C hex
floats together with the fp32 evaluation's maximum relative error on a dense
grid; the kernel's constants are these values, and
``tests/test_exp2_poly.py`` checks both the match and the bound.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
NODES = 512
LAWSON_ITERS = 200


def fit(degree: int = DEGREE, nodes: int = NODES, iters: int = LAWSON_ITERS) -> np.ndarray:
    """Coefficients c0..c_degree (fp64) of the relative-error minimax
    approximation of 2^f on [-1/2, 1/2], by Lawson's iteration."""
    k = np.arange(nodes)
    f = 0.5 * np.cos((2 * k + 1) * np.pi / (2 * nodes))  # Chebyshev nodes of [-1/2, 1/2]
    y = np.exp2(f)
    A = np.vander(f, degree + 1, increasing=True) / y[:, None]  # relative residual: (p(f) - y) / y
    b = np.ones_like(f)
    w = np.full(nodes, 1.0 / nodes)
    c = None
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], b * sw, rcond=None)
        err = np.abs(A @ c - b)
        w = w * err
        w = w / w.sum()
    return c


def coefficients_f32() -> np.ndarray:
    """The fitted coefficients rounded to fp32 (what the kernel holds)."""
    return fit().astype(np.float32)


def c_hex(v: np.float32) -> str:
    """C99 hex-float literal of an fp32 value (e.g. 0x1.62f31ap-1f)."""
    m, e = np.frexp(np.float64(v))  # v = m * 2^e, m in [0.5, 1)
    m, e = m * 2.0, e - 1
    frac = int(round((m - 1.0) * (1 << 24)))  # 23 fraction bits, padded to 6 hex digits
    return f"0x1.{frac:06x}p{e}f"


def horner_f32(c: np.ndarray, f: np.ndarray) -> np.ndarray:
    """Horner evaluation of the cubic at fp32 f with one fp32 rounding per
    step, as the kernel's FMAs do (each a*b+c is formed exactly in fp64,
    since a*b of two fp32 values has at most 48 significant bits, then
    rounded to fp32; this double rounding can differ from a fused
    single rounding by one ulp, rarely)."""
    c = [np.float32(v) for v in c]
    f64 = f.astype(np.float64)
    r = np.float32(c[3])
    r = (np.float64(r) * f64 + np.float64(c[2])).astype(np.float32)
    r = (r.astype(np.float64) * f64 + np.float64(c[1])).astype(np.float32)
    r = (r.astype(np.float64) * f64 + np.float64(c[0])).astype(np.float32)
    return r


def exp2_emulated(x: np.ndarray, c: np.ndarray) -> np.ndarray:
    """The kernel's 2^x in numpy fp32: clamp at -125, n = round(x) by the
    1.5 * 2^23 shift, f = x - n, the cubic, then n added to the exponent
    field as an int32 (wrapping) add of n << 23."""
    shift = np.float32(12582912.0)
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-125.0))
    t = (x + shift).astype(np.float32)
    nr = (shift - t).astype(np.float32)  # -n, exact
    fr = (x + nr).astype(np.float32)     # x - n, exact
    p = horner_f32(c, fr)
    pb = p.view(np.int32).astype(np.int64)
    tb = t.view(np.int32).astype(np.int64)
    out = (pb + (tb << 23)) & 0xFFFFFFFF
    return out.astype(np.uint32).view(np.float32)


def max_rel_error(c: np.ndarray, lo: float = -125.0, hi: float = 8.0, n: int = 2_000_001) -> float:
    """Maximum relative error of :func:`exp2_emulated` against fp64 2^x on a
    uniform grid of [lo, hi] (the kernel's range: the clamp below, the
    lazily rebased running max above)."""
    x = np.linspace(lo, hi, n).astype(np.float32)
    got = exp2_emulated(x, c).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    return float(np.max(np.abs(got - ref) / ref))


if __name__ == "__main__":
    c = coefficients_f32()
    print("c0..c3 =", ", ".join(c_hex(v) for v in c))
    print("max relative error on [-125, 8] (fp32 evaluation): %.3e" % max_rel_error(c))
