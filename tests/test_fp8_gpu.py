"""GPU parity of the FP8 prefill path against the oracle.

attn_quantize_fp8: codes bit-exact and scales equal to the oracle's block
quantisation (the code decision is taken in fp32 on both sides); with
incoherent processing the rotation is a sum of 128 fp32 terms whose rounding
depends on the order of additions, so codes may differ only where the exact
value sits within fp32 rounding of a rounding boundary, and scales agree to
1e-5.  attn_fwd_fp8: against the fp64 oracle of exact attention on the
dequantised Q and K (inputs quantised by the oracle on the CPU) and bf16 V,
with the bf16 tolerances (max 2e-2, mean 2e-3, LSE 1e-3): the tensor core
multiplies e4m3 values exactly and accumulates in fp32.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from oracle import fp8 as F
from tests._parity import check_close, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import online_softmax_paged_b200 as osp
    osp.load()


def _osp():
    import online_softmax_paged_b200 as osp
    return osp


def _x(shape, seed, scales=None):
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randn(shape, generator=g)
    if scales is not None:
        x = x * scales
    return x.to(torch.bfloat16)


def _near_boundary(v, rel=1e-5):
    mids = (F.E4M3_GRID[:-1] + F.E4M3_GRID[1:]) / 2
    a = np.abs(v)
    i = np.clip(np.searchsorted(mids, a), 1, len(mids) - 1)
    d = np.minimum(np.abs(a - mids[i - 1]), np.abs(a - mids[i]))
    return d <= rel * np.maximum(a, 2.0 ** -9)


def test_quantize_bit_exact_plain():
    osp = _osp()
    x = _x((2, 3, 300, 128), 1, torch.tensor([0.01, 1.0, 40.0]).view(1, 3, 1, 1))
    x[1, 0, 128:256] = 0  # all-zero block
    x[0, 2, 5, 7] = 3.0e4  # a large outlier
    codes, scales = osp.attn_quantize_fp8(x.cuda())
    torch.cuda.synchronize()
    c_ref, s_ref = F.quantize_blocks(x.float().numpy(), 128)
    np.testing.assert_array_equal(codes.cpu().numpy(), F.e4m3_code(c_ref))
    np.testing.assert_array_equal(scales.cpu().numpy(), s_ref)
    # the bytes are torch's float8_e4m3fn of the same values
    assert torch.equal(codes.view(torch.float8_e4m3fn).float().cpu(), torch.from_numpy(c_ref).float())


def test_quantize_rotated():
    osp = _osp()
    x = _x((2, 2, 260, 128), 2)
    s = W.hadamard_signs(128, seed=3)
    codes, scales = osp.attn_quantize_fp8(x.cuda(), signs=s.cuda())
    torch.cuda.synchronize()
    xf = x.float().numpy()
    c_ref, s_ref = F.quantize_blocks(xf, 128, signs=s.numpy())
    np.testing.assert_allclose(scales.cpu().numpy(), s_ref, rtol=1e-5)
    got = F.e4m3_decode(codes.cpu().numpy())
    diff = got != c_ref
    # the pre-rounding values of the oracle (fp32 y * r) at the mismatches
    y = F.rotate(xf, s.numpy()).astype(np.float32)
    assert diff.mean() < 1e-3, diff.mean()
    if diff.any():
        idx = np.argwhere(diff)
        for (a, h, n, k) in idx[:200]:
            blk = n // 128
            blk_vals = y[a, h, blk * 128:(blk + 1) * 128]
            r = np.float32(448.0) / np.abs(blk_vals).max()
            assert _near_boundary(np.float32(y[a, h, n, k] * r)), (a, h, n, k)
            assert abs(got[a, h, n, k] - c_ref[a, h, n, k]) <= np.diff(F.E4M3_GRID).max()
    # dequantised rows stay within half an e4m3 step of the exact rotation / sqrt(d)
    deq = F.dequantize_blocks(got, scales.cpu().numpy())
    exact = F.rotate(xf, s.numpy()) / np.sqrt(128)
    sc = np.repeat(scales.cpu().numpy().astype(np.float64), 128, axis=-1)[..., :260, None]
    assert np.all(np.abs(deq - exact) <= 2.0 ** -4 * np.abs(exact) + 2.0 ** -10 * sc + 1e-5 * np.abs(exact) + 1e-7)


def _fp8_inputs(B, H, N, seed, rotate, mult=1.0):
    inp = W.dense_inputs(B, H, N, 128, dtype=torch.bfloat16, mult=mult, seed=seed, device="cpu")
    s = W.hadamard_signs(128, seed=seed + 100).numpy() if rotate else None
    qc, qs = F.quantize_blocks(inp["Q"].float().numpy(), 128, signs=s)
    kc, ks = F.quantize_blocks(inp["K"].float().numpy(), 128, signs=s)
    dev = dict(q8=torch.from_numpy(F.e4m3_code(qc)).cuda(), q_scale=torch.from_numpy(qs).cuda(),
               k8=torch.from_numpy(F.e4m3_code(kc)).cuda(), k_scale=torch.from_numpy(ks).cuda(), V=inp["V"].cuda())
    ref = dict(Q=F.dequantize_blocks(qc, qs), K=F.dequantize_blocks(kc, ks), V=to64(inp["V"]), scale=inp["scale"])
    return inp, dev, ref


@pytest.mark.parametrize("B,H,N,causal,rotate", [(1, 2, 128, False, False), (1, 2, 300, True, False),
                                                 (2, 3, 700, True, True), (1, 2, 513, False, True),
                                                 (1, 1, 1, True, False), (1, 2, 2000, True, False)])
def test_fp8_attention_parity(B, H, N, causal, rotate):
    osp = _osp()
    _, dev, ref = _fp8_inputs(B, H, N, seed=B * 100 + N, rotate=rotate)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O, LSE = osp.attn_fwd_fp8(dev["q8"], dev["q_scale"], dev["k8"], dev["k_scale"], dev["V"], causal=causal,
                              scale=ref["scale"], err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    O_ref, L_ref = oracle.attention_dense(ref["Q"], ref["K"], ref["V"], causal, ref["scale"])
    check_close(O, LSE, O_ref, L_ref, torch.bfloat16, f"fp8 B={B} H={H} N={N} causal={causal} rot={rotate}")


def test_fp8_prefill_2k_full_size():
    """The causal prefill 2k workload (B=4 H=16 N=2048) with e4m3 Q/K and
    incoherent processing: four heads in full against the oracle."""
    osp = _osp()
    _, dev, ref = _fp8_inputs(4, 16, 2048, seed=0, rotate=True)
    O, LSE = osp.attn_fwd_fp8(dev["q8"], dev["q_scale"], dev["k8"], dev["k_scale"], dev["V"], causal=True,
                              scale=ref["scale"])
    torch.cuda.synchronize()
    assert torch.isfinite(O.float()).all() and torch.isfinite(LSE).all()
    heads = [(0, 0), (1, 7), (2, 3), (3, 15)]
    O_ref, L_ref = oracle.attention_dense(ref["Q"], ref["K"], ref["V"], True, ref["scale"], heads=heads)
    for b, h in heads:
        check_close(O[b, h], LSE[b, h], O_ref[b, h], L_ref[b, h], torch.bfloat16, f"fp8 2k head {(b, h)}")


@pytest.mark.parametrize("rotate", [False, True])
def test_quantize_then_attend_end_to_end(rotate):
    """GPU quantisation followed by the FP8 kernel equals the oracle pipeline
    (oracle quantisation, exact attention on the dequantised operands), and
    stays close to exact bf16 attention on the unquantised inputs."""
    osp = _osp()
    inp, _, ref = _fp8_inputs(1, 4, 640, seed=5, rotate=rotate)
    s = W.hadamard_signs(128, seed=105).cuda() if rotate else None
    q8, qs = osp.attn_quantize_fp8(inp["Q"].cuda(), signs=s)
    k8, ks = osp.attn_quantize_fp8(inp["K"].cuda(), signs=s)
    O, LSE = osp.attn_fwd_fp8(q8, qs, k8, ks, inp["V"].cuda(), causal=True, scale=inp["scale"])
    torch.cuda.synchronize()
    O_ref, L_ref = oracle.attention_dense(ref["Q"], ref["K"], ref["V"], True, ref["scale"])
    check_close(O, LSE, O_ref, L_ref, torch.bfloat16, f"quantise+attend rot={rotate}")
    O_x, _ = oracle.attention_dense(to64(inp["Q"]), to64(inp["K"]), to64(inp["V"]), True, inp["scale"])
    assert np.abs(to64(O) - O_x).mean() < 2e-2


def test_fp8_rejects_other_head_dims():
    osp = _osp()
    x = torch.zeros((1, 1, 128, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(osp.AttnError):
        osp.attn_quantize_fp8(x)


def test_fp8_many_units_per_cta_ragged():
    """FP8 with B=2 H=90 N=300 (360 units over at most 148 CTAs, empty upper
    tiles included) against the oracle on the dequantised operands."""
    osp = _osp()
    _, dev, ref = _fp8_inputs(2, 90, 300, seed=22, rotate=True)
    O, LSE = osp.attn_fwd_fp8(dev["q8"], dev["q_scale"], dev["k8"], dev["k_scale"], dev["V"], causal=True,
                              scale=ref["scale"])
    torch.cuda.synchronize()
    O_ref, L_ref = oracle.attention_dense(ref["Q"], ref["K"], ref["V"], True, ref["scale"])
    check_close(O, LSE, O_ref, L_ref, torch.bfloat16, "fp8 many units")
