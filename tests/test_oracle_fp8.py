"""Pins of the FP8 (e4m3) quantisation oracle against things other than
itself: PyTorch's float8_e4m3fn conversion (an independent implementation of
the format), the format's own definition (grid size, extremes, ties to even,
saturation), the Hadamard matrix's orthogonality, the quantisation error
bound, and the method-level claim that block scales with incoherent
processing lose less accuracy than one scale per head on inputs with
outliers ("一文掌握大模型推理加速：FlashAttention与PagedAttention技术详解",
§二 "FlashAttention-3改进" and "性能提升")."""
import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import fp8 as F


def test_grid_definition():
    g = F.E4M3_GRID
    assert len(g) == 127  # codes 0x00 .. 0x7e
    assert g[0] == 0 and g[1] == 2.0 ** -9 and g[-1] == 448.0
    assert np.all(np.diff(g) > 0)
    assert g[8] == 2.0 ** -6  # smallest normal
    # the spacing doubles at each power of two from the first normal binade on
    assert np.allclose(np.diff(g[8:16]), 2.0 ** -9) and np.allclose(np.diff(g[16:24]), 2.0 ** -8)


def test_round_matches_torch_float8():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.05, 1, 30, 200)])
    x = x[np.abs(x) <= 448].astype(np.float32)
    x = np.concatenate([x, F.E4M3_GRID.astype(np.float32), -F.E4M3_GRID.astype(np.float32)])
    t = torch.from_numpy(x).to(torch.float8_e4m3fn)
    np.testing.assert_array_equal(F.e4m3_round(x), t.float().numpy().astype(np.float64))
    np.testing.assert_array_equal(F.e4m3_code(F.e4m3_round(x)), t.view(torch.uint8).numpy())
    np.testing.assert_array_equal(F.e4m3_decode(t.view(torch.uint8).numpy()), t.float().numpy())


def test_ties_to_even_and_saturation():
    g = F.E4M3_GRID
    mid = (g[:-1] + g[1:]) / 2
    r = F.e4m3_round(mid)
    lo_even = (np.arange(len(g) - 1) % 2 == 0)
    np.testing.assert_array_equal(r, np.where(lo_even, g[:-1], g[1:]))
    assert F.e4m3_round(1000.0) == 448.0 and F.e4m3_round(-1e30) == -448.0 and F.e4m3_round(449.0) == 448.0
    assert F.e4m3_round(2.0 ** -10) == 0.0 and F.e4m3_round(2.0 ** -10 * 1.0001) == 2.0 ** -9
    assert np.isnan(F.e4m3_round(np.nan))


def test_hadamard_rotation_preserves_products():
    for d in (1, 2, 8, 64, 128):
        H = F.hadamard(d)
        np.testing.assert_array_equal(H @ H.T, d * np.eye(d))
        np.testing.assert_array_equal(H, H.T)
    rng = np.random.default_rng(1)
    s = rng.choice([-1.0, 1.0], 128)
    q, k = rng.standard_normal((5, 128)), rng.standard_normal((7, 128))
    np.testing.assert_allclose(F.rotate(q, s) @ F.rotate(k, s).T, 128 * q @ k.T, rtol=1e-12, atol=1e-10)
    with pytest.raises(ValueError):
        F.hadamard(96)


@pytest.mark.parametrize("rot", [False, True])
def test_quantize_error_bound_and_block_max(rot):
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((3, 300, 128)) * rng.uniform(0.01, 5, (3, 1, 1))).astype(np.float32)
    x[1, 128:256] = 0  # an all-zero block
    s = rng.choice([-1.0, 1.0], 128) if rot else None
    codes, scales = F.quantize_blocks(x, 128, signs=s)
    assert codes.shape == x.shape and scales.shape == (3, 3)
    assert np.abs(codes).max() == 448.0
    assert scales[1, 1] == 1.0 and np.all(codes[1, 128:256] == 0)
    y = F.rotate(x, s) / np.sqrt(128) if rot else x.astype(np.float64)
    deq = F.dequantize_blocks(codes, scales)
    sc = np.repeat(scales.astype(np.float64), 128, axis=-1)[..., :300, None]
    # half an e4m3 step: 2^-4 relative for normal codes, 2^-10 in code units below 2^-6,
    # plus the fp32 rounding of the scale and of y * r
    bound = 2.0 ** -4 * np.abs(y) + 2.0 ** -10 * sc + 1e-6 * np.abs(y)
    assert np.all(np.abs(deq - y) <= bound)
    # the dequantised rotated operands still give q k^T (rotation folded into the scales)
    if rot:
        k = rng.standard_normal((1, 200, 128)).astype(np.float32)
        kc, ks = F.quantize_blocks(k, 128, signs=s)
        approx = deq[0] @ F.dequantize_blocks(kc, ks)[0].T
        exact = x[0].astype(np.float64) @ k[0].astype(np.float64).T
        assert np.abs(approx - exact).max() < 0.25 * np.abs(exact).max()


def test_incoherent_processing_reduces_fp8_attention_error():
    """Inputs N(0,1) with 0.1% outliers of N(0,100): exact attention on e4m3
    Q/K quantised with one scale per head and no rotation has a larger error
    than with 128-row block scales and incoherent processing.  (The pages'
    2.6x is for an FP8 attention that also quantises P and V; with Q and K
    alone the reduction measured here is about 1.4x.)"""
    rng = np.random.default_rng(3)
    N, d = 512, 128

    def draw():
        x = rng.standard_normal((N, d))
        m = rng.random((N, d)) < 1e-3
        x[m] += rng.standard_normal(m.sum()) * 10
        return x.astype(np.float32)

    s = rng.choice([-1.0, 1.0], d)
    errs_base, errs_ip = [], []
    for _ in range(3):
        q, k, v = draw(), draw(), draw()
        o_ref, _ = A.attention_head(q.astype(np.float64), k.astype(np.float64), v.astype(np.float64), True,
                                    d ** -0.5)
        qb = F.dequantize_blocks(*F.quantize_blocks(q[None], N), N)[0]
        kb = F.dequantize_blocks(*F.quantize_blocks(k[None], N), N)[0]
        qi = F.dequantize_blocks(*F.quantize_blocks(q[None], 128, signs=s))[0]
        ki = F.dequantize_blocks(*F.quantize_blocks(k[None], 128, signs=s))[0]
        o_b, _ = A.attention_head(qb, kb, v.astype(np.float64), True, d ** -0.5)
        # rotated operands: (q D H / sqrt d)(k D H / sqrt d)^T = q k^T
        o_i, _ = A.attention_head(qi, ki, v.astype(np.float64), True, d ** -0.5)
        errs_base.append(np.sqrt(np.mean((o_b - o_ref) ** 2)))
        errs_ip.append(np.sqrt(np.mean((o_i - o_ref) ** 2)))
    assert np.mean(errs_ip) * 1.2 < np.mean(errs_base), (errs_ip, errs_base)


def test_planted_mistakes_fail():
    """A quantiser that rounds toward zero, or uses the other e4m3 variant's
    bias 8 (largest value 240, smallest 2^-10), disagrees with the
    independent conversion."""
    rng = np.random.default_rng(4)
    x = np.concatenate([rng.standard_normal(5000) * 20, rng.uniform(240, 448, 50), rng.uniform(0, 2 ** -6, 50)])
    x = x.astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).float().numpy()
    assert np.array_equal(F.e4m3_round(x), ref)
    g = F.E4M3_GRID
    trunc = np.copysign(g[np.searchsorted(g, np.abs(x), side="right") - 1], x)
    assert not np.array_equal(trunc, ref)
    bias8 = F.e4m3_round(x * 2.0) / 2.0  # every value one binade lower
    assert not np.array_equal(bias8, ref)
