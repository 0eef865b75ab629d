"""The exponential the bf16 prefill softmax evaluates on the FMA pipe.

Part of every unmasked score row is exponentiated by a cubic instead of the
special-function unit (2^x = 2^round(x) * p(x - round(x))).  These tests pin
it three ways:

* the committed fit (online_softmax_paged_b200/exp2_poly_fit.py: Chebyshev
  nodes, Lawson's iteration towards the relative-error minimax, rounded to
  fp32) reproduces the four constants the device code holds, read from
  csrc/softmax_math.cuh;
* a numpy fp32 restatement of the device steps (clamp, shift rounding,
  Horner, exponent add) stays within the stated bound, relative error
  <= 7.5e-5 against fp64 2^x on a dense grid of [-125, 8] (the clamp below;
  the lazily rebased running max lets x reach +8 above);
* on the GPU, the device function itself, run through the C ABI self-test
  entry point, meets the same bound and agrees with the restatement to one
  ulp (the restatement rounds each FMA twice, fp64 then fp32).
"""
import os
import re

import numpy as np
import pytest
import torch

from online_softmax_paged_b200 import exp2_poly_fit as F

BOUND = 7.5e-5
HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "online_softmax_paged_b200",
                      "csrc", "softmax_math.cuh")


def _device_constants():
    src = open(HEADER).read()
    vals = {}
    for name in ("c0", "c1", "c2", "c3"):
        m = re.search(r"\b%s = (0x[0-9a-fA-F.]+p[-+]?\d+)f" % name, src)
        assert m, f"{name} not found in softmax_math.cuh"
        vals[name] = float.fromhex(m.group(1))
    return np.array([vals["c0"], vals["c1"], vals["c2"], vals["c3"]], dtype=np.float32)


def test_fit_reproduces_device_constants():
    fitted = F.coefficients_f32()
    dev = _device_constants()
    assert fitted.tobytes() == dev.tobytes(), (F.c_hex(fitted[0]), F.c_hex(fitted[1]), F.c_hex(fitted[2]),
                                              F.c_hex(fitted[3]))
    # the printed literals round-trip
    for v in fitted:
        assert np.float32(float.fromhex(F.c_hex(v)[:-1])) == v


def test_fit_is_near_minimax():
    """Lawson's iteration equioscillates: the relative error of the fp64 fit
    reaches its maximum with alternating signs at degree + 2 points."""
    c = F.fit()
    f = np.linspace(-0.5, 0.5, 200001)
    e = np.polyval(c[::-1], f) / np.exp2(f) - 1.0
    emax = np.abs(e).max()
    assert emax < BOUND
    # local extrema of |e| above 0.99 * max: at least 5 with alternating signs
    idx = [i for i in range(1, len(f) - 1) if abs(e[i]) >= abs(e[i - 1]) and abs(e[i]) >= abs(e[i + 1])]
    idx = [0] + idx + [len(f) - 1]
    peaks = [i for i in idx if abs(e[i]) > 0.99 * emax]
    signs = np.sign(e[peaks])
    assert len(peaks) >= 5
    assert all(signs[k] != signs[k + 1] for k in range(len(signs) - 1))


def test_emulated_bound_on_kernel_range():
    c = _device_constants()
    assert F.max_rel_error(c, -125.0, 8.0, 4_000_001) <= BOUND


def test_emulated_special_points():
    c = _device_constants()
    x = np.array([0.0, 1.0, -1.0, 8.0, -125.0, -0.5, 0.5, -124.5, 3.25], dtype=np.float32)
    got = F.exp2_emulated(x, c).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert (np.abs(got / ref - 1.0) <= BOUND).all()
    # below the clamp the result is 2^-125 (normal, and ~0 next to l >= 1)
    low = F.exp2_emulated(np.array([-126.0, -1e4, -np.inf], dtype=np.float32), c)
    assert np.allclose(low.astype(np.float64), F.exp2_emulated(np.array([-125.0], dtype=np.float32), c)[0])
    assert (low > 0).all() and np.isfinite(low).all()


def test_planted_wrong_constant_fails_bound():
    c = _device_constants().copy()
    c[2] = np.float32(c[2] * 1.01)  # a 1 % error in the quadratic term
    assert F.max_rel_error(c, -125.0, 8.0, 200_001) > BOUND


@pytest.mark.gpu
def test_device_polynomial_within_bound():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import online_softmax_paged_b200 as osp
    x = torch.linspace(-125.0, 8.0, 4_000_001, dtype=torch.float64).float()
    x = torch.cat([x, torch.tensor([0.0, 1.0, -1.0, 0.5, -0.5, -126.0, -1e4], dtype=torch.float32)])
    y = osp.attn_selftest_exp2_poly(x.cuda())
    torch.cuda.synchronize()
    got = y.cpu().numpy()
    xs = x.numpy()
    ref = np.exp2(np.maximum(xs, -125.0).astype(np.float64))
    rel = np.abs(got.astype(np.float64) / ref - 1.0)
    assert rel.max() <= BOUND, rel.max()
    emu = F.exp2_emulated(xs, _device_constants())
    ulps = np.abs(got.view(np.int32).astype(np.int64) - emu.view(np.int32).astype(np.int64))
    assert ulps.max() <= 1
    assert (ulps == 0).mean() > 0.999
