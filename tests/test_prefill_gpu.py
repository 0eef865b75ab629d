"""GPU parity of the dense entry point (attn_fwd) against the fp64 oracle.

bf16 runs the tcgen05 kernel, fp32 the CUDA-core kernel; both through the
C ABI.  Shapes span several 128-row / 128-key tiles with ragged tails; the
full-size prefill workloads are checked on sampled heads and rows the oracle
computes one by one, and through closed-form properties at full size.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W
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


def _run(inp, err=None):
    O, LSE = _osp().attn_fwd(inp["Q"], inp["K"], inp["V"], causal=inp["causal"], scale=inp["scale"], err_flag=err)
    torch.cuda.synchronize()
    return O, LSE


def _full_oracle(inp):
    return oracle.attention_dense(to64(inp["Q"]), to64(inp["K"]), to64(inp["V"]), inp["causal"], inp["scale"])


def test_fp32_small_config():
    """Dense fp32, non-causal, B=1 H=2 N=128 d=64, seed 0 (max |dO| <= 1e-4)."""
    inp = W.dense_inputs(1, 2, 128, 64, dtype=torch.float32, seed=0, device="cuda")
    O, LSE = _run(inp)
    O_ref, L_ref = _full_oracle(inp)
    check_close(O, LSE, O_ref, L_ref, torch.float32, "fp32 1x2x128x64")


@pytest.mark.parametrize("B,H,N,d,causal", [
    (1, 2, 77, 64, True), (2, 1, 200, 128, False), (1, 3, 129, 128, True), (1, 1, 1, 64, False),
    (1, 2, 300, 64, True),
])
def test_fp32_shapes(B, H, N, d, causal):
    inp = W.dense_inputs(B, H, N, d, dtype=torch.float32, seed=1, device="cuda", causal=causal)
    O, LSE = _run(inp)
    O_ref, L_ref = _full_oracle(inp)
    check_close(O, LSE, O_ref, L_ref, torch.float32, f"fp32 {B}x{H}x{N}x{d} causal={causal}")


BF16_SHAPES = [
    (1, 1, 1, 128, True), (1, 1, 1, 128, False), (1, 1, 128, 128, True), (1, 1, 256, 128, True),
    (1, 1, 257, 128, False), (1, 2, 300, 128, False), (1, 2, 300, 128, True), (2, 3, 513, 64, True),
    (2, 3, 513, 64, False), (1, 2, 1000, 128, True), (3, 2, 640, 128, True), (1, 1, 1100, 64, False),
]


@pytest.mark.parametrize("B,H,N,d,causal", BF16_SHAPES)
def test_bf16_shapes(B, H, N, d, causal):
    inp = W.dense_inputs(B, H, N, d, dtype=torch.bfloat16, seed=2, device="cuda", causal=causal)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O, LSE = _run(inp, err)
    O_ref, L_ref = _full_oracle(inp)
    check_close(O, LSE, O_ref, L_ref, torch.bfloat16, f"bf16 {B}x{H}x{N}x{d} causal={causal}")
    assert int(err.item()) == 0


def test_bf16_large_scores_stay_exact():
    """Scores spanning tens of nats in one row: the reference max moves, the
    O accumulator is rescaled, and the result still matches."""
    inp = W.dense_inputs(1, 2, 700, 128, dtype=torch.bfloat16, seed=3, device="cuda", causal=True)
    inp["Q"] = (inp["Q"].float() * 4).to(torch.bfloat16)
    O, LSE = _run(inp)
    O_ref, L_ref = _full_oracle(inp)
    check_close(O, LSE, O_ref, L_ref, torch.bfloat16, "bf16 large scores")


@pytest.mark.parametrize("causal", [True, False])
def test_bf16_late_score_jump(causal):
    """Keys from position 384 on score ~28 nats (~40 in log2 units) above the
    first key tile: the reference max set by the first tile is too low by
    more than 2^32, so the kernel must redo those tiles with their own max."""
    inp = W.dense_inputs(1, 2, 900, 128, dtype=torch.bfloat16, seed=11, device="cuda", causal=causal)
    Q, K = inp["Q"].clone(), inp["K"].clone()
    Q[..., 0] = 2.0
    K[..., 384:, 0] = 160.0
    inp["Q"], inp["K"] = Q.contiguous(), K.contiguous()
    O, LSE = _run(inp)
    O_ref, L_ref = _full_oracle(inp)
    # the jump is really there: rows past 384 see scores ~28 nats above the first tile's
    assert L_ref[..., 500:].min() > 25.0
    if causal:
        assert L_ref[..., :384].max() < 15.0
    check_close(O, LSE, O_ref, L_ref, torch.bfloat16, f"late score jump causal={causal}")


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("keys", ["tile", "poly_column", "sfu_column", "both_halves"])
def test_bf16_extreme_score_jump(causal, keys):
    """Keys that score ~141 nats (~204 in log2 units) above the rest: a whole
    key tile from position 384 on, or single keys at positions 394 and 906
    (columns 10 of their tiles, exponentiated on the FMA pipe) or 384 (column
    0, special-function unit), or one in each 128-row half of a query block.
    Exponentials of those tiles against the running max carried from earlier
    tiles would overflow fp32, so the running max must move to the new tile's
    row max before any of them is taken, whichever unit (special-function or
    FMA pipe) takes it.  The result is still the plain definition's."""
    inp = W.dense_inputs(1, 2, 1000, 128, dtype=torch.bfloat16, seed=12, device="cuda", causal=causal)
    Q, K = inp["Q"].clone(), inp["K"].clone()
    Q[..., 0] = 4.0
    sel = {"tile": slice(384, 512), "poly_column": [394, 906], "sfu_column": [384],
           "both_halves": [394, 522]}[keys]
    K[..., sel, 0] = 400.0
    inp["Q"], inp["K"] = Q.contiguous(), K.contiguous()
    O, LSE = _run(inp)
    O_ref, L_ref = _full_oracle(inp)
    assert L_ref[..., 600:].min() > 130.0
    check_close(O, LSE, O_ref, L_ref, torch.bfloat16, f"extreme score jump {keys} causal={causal}")


def test_prefill_2k_causal_full_size():
    """B=4 H=16 N=2048 d=128 causal bf16, seed 0: the launch the bench times.
    Four (b, h) heads against the oracle in full; every head for finiteness."""
    inp = W.dense_inputs(device="cuda", seed=0, **{k: v for k, v in W.PREFILL_CAUSAL_2K.items() if k != "mult"})
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O, LSE = _run(inp, err)
    assert int(err.item()) == 0
    assert torch.isfinite(O.float()).all() and torch.isfinite(LSE).all()
    heads = [(0, 0), (1, 7), (2, 3), (3, 15)]
    O_ref, L_ref = oracle.attention_dense(to64(inp["Q"]), to64(inp["K"]), to64(inp["V"]), True, inp["scale"],
                                          heads=heads)
    for b, h in heads:
        check_close(O[b, h], LSE[b, h], O_ref[b, h], L_ref[b, h], torch.bfloat16, f"2k head {(b, h)}")


def test_prefill_16k_causal_sampled():
    """B=1 H=32 N=16384 d=128 causal bf16 (values x0.5), seed 0: one full head
    plus sampled rows of three others, each row computed alone by the oracle
    (causal row i = one query against keys 0..i)."""
    cfg = W.PREFILL_CAUSAL_16K
    inp = W.dense_inputs(cfg["B"], cfg["H"], cfg["N"], cfg["d"], dtype=cfg["dtype"], mult=cfg["mult"], seed=0,
                         device="cuda", causal=True)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O, LSE = _run(inp, err)
    assert int(err.item()) == 0
    h = 5
    Qh, Kh, Vh = (to64(inp[k][0, h]) for k in ("Q", "K", "V"))
    O_ref, L_ref = oracle.attention_head(Qh, Kh, Vh, True, inp["scale"])
    check_close(O[0, h], LSE[0, h], O_ref, L_ref, torch.bfloat16, "16k full head")
    rows = [0, 1, 127, 128, 255, 256, 1000, 4095, 8191, 8192, 12345, 16383]
    for h in (0, 17, 31):
        Qh, Kh, Vh = (to64(inp[k][0, h]) for k in ("Q", "K", "V"))
        Og, Lg = to64(O[0, h]), to64(LSE[0, h])
        for i in rows:
            o, l = oracle.attention_head(Qh[i:i + 1], Kh[:i + 1], Vh[:i + 1], False, inp["scale"])
            assert np.abs(Og[i] - o[0]).max() <= 2e-2, (h, i)
            assert abs(Lg[i] - l[0]) <= 1e-3, (h, i)


def test_properties_full_size():
    """Closed forms at the 2k workload size: Q = 0 gives LSE_i = ln(i + 1) and
    O_i = prefix mean of V; uniform V gives O = v."""
    B, H, N, d = 4, 16, 2048, 128
    inp = W.dense_inputs(B, H, N, d, dtype=torch.bfloat16, seed=4, device="cuda", causal=True)
    inp["Q"] = torch.zeros_like(inp["Q"])
    O, LSE = _run(inp)
    i = torch.arange(N, device="cuda", dtype=torch.float64)
    assert (LSE.double() - torch.log(i + 1)).abs().max().item() <= 1e-3
    pm = torch.cumsum(inp["V"].double(), dim=2) / (i + 1)[None, None, :, None]
    assert (O.double() - pm).abs().max().item() <= 2e-2
    v = torch.randn(d, device="cuda").to(torch.bfloat16)
    inp = W.dense_inputs(B, H, N, d, dtype=torch.bfloat16, seed=5, device="cuda", causal=True)
    inp["V"] = v.expand(B, H, N, d).contiguous()
    O, _ = _run(inp)
    assert (O.double() - v.double()).abs().max().item() <= 2e-2


def test_outputs_written_exactly_in_place():
    """Canary: the kernel writes O and LSE completely and nothing past them."""
    osp = _osp()
    B, H, N, d = 1, 3, 333, 128
    inp = W.dense_inputs(B, H, N, d, dtype=torch.bfloat16, seed=6, device="cuda", causal=True)
    n_o, n_l = B * H * N * d, B * H * N
    big_o = torch.full((n_o + 4096,), float("nan"), dtype=torch.bfloat16, device="cuda")
    big_l = torch.full((n_l + 1024,), float("nan"), dtype=torch.float32, device="cuda")
    O = big_o[:n_o].view(B, H, N, d)
    L = big_l[:n_l].view(B, H, N)
    osp.attn_fwd(inp["Q"], inp["K"], inp["V"], O=O, LSE=L, causal=True)
    torch.cuda.synchronize()
    assert torch.isnan(big_o[n_o:].float()).all() and torch.isnan(big_l[n_l:]).all()
    assert torch.isfinite(O.float()).all() and torch.isfinite(L).all()


def test_deterministic():
    inp = W.dense_inputs(2, 4, 900, 128, dtype=torch.bfloat16, seed=7, device="cuda", causal=True)
    O1, L1 = _run(inp)
    O2, L2 = _run(inp)
    assert torch.equal(O1, O2) and torch.equal(L1, L2)


def test_fp32_is_not_tf32():
    """fp32 results keep fp32 accuracy (a TF32 product would miss 1e-4)."""
    inp = W.dense_inputs(1, 2, 256, 128, dtype=torch.float32, seed=8, device="cuda", causal=False)
    inp["Q"] = inp["Q"] * 3
    O, LSE = _run(inp)
    O_ref, L_ref = _full_oracle(inp)
    assert np.abs(to64(O) - O_ref).max() <= 1e-4


@pytest.mark.parametrize("causal", [True, False])
def test_bf16_many_units_per_cta_ragged(causal):
    """B=2 H=100 N=300: 400 units over at most 148 CTAs, so each CTA walks
    two or three units, and every second unit's upper query tile has no rows
    (it is skipped by the producer, the MMA issuer and the O staging order)."""
    inp = W.dense_inputs(2, 100, 300, 128, dtype=torch.bfloat16, seed=21, device="cuda", causal=causal)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O, LSE = _run(inp, err)
    assert int(err.item()) == 0
    O_ref, L_ref = oracle.attention_dense(to64(inp["Q"]), to64(inp["K"]), to64(inp["V"]), causal, inp["scale"])
    check_close(O, LSE, O_ref, L_ref, torch.bfloat16, f"many units causal={causal}")
