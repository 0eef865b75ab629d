"""Shared tolerance checks for the GPU parity tests.

Tolerances (stated for this path; elementwise against the fp64 oracle on the
same bf16/fp32-rounded inputs):
  bf16: max |dO| <= 2e-2, mean |dO| <= 2e-3
  fp32: max |dO| <= 1e-4
  all : max |dLSE| <= 1e-3
"""
import numpy as np
import torch

BF16_MAX, BF16_MEAN, F32_MAX, LSE_MAX = 2e-2, 2e-3, 1e-4, 1e-3


def to64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_close(O_gpu, LSE_gpu, O_ref, LSE_ref, dtype, what=""):
    O = to64(O_gpu) if isinstance(O_gpu, torch.Tensor) else O_gpu
    L = to64(LSE_gpu) if isinstance(LSE_gpu, torch.Tensor) else LSE_gpu
    assert O.shape == O_ref.shape, (O.shape, O_ref.shape)
    assert np.isfinite(O).all(), f"{what}: non-finite O"
    fin = np.isfinite(LSE_ref)
    assert (np.isfinite(L) == fin).all(), f"{what}: LSE finiteness differs"
    assert (L[~fin] == LSE_ref[~fin]).all(), f"{what}: LSE -inf mismatch"
    dO = np.abs(O - O_ref)
    dL = np.abs(L[fin] - LSE_ref[fin]) if fin.any() else np.zeros(1)
    if dtype == torch.float32:
        assert dO.max() <= F32_MAX, f"{what}: max|dO| {dO.max():.3e} > {F32_MAX}"
    else:
        assert dO.max() <= BF16_MAX, f"{what}: max|dO| {dO.max():.3e} > {BF16_MAX}"
        assert dO.mean() <= BF16_MEAN, f"{what}: mean|dO| {dO.mean():.3e} > {BF16_MEAN}"
    assert dL.max() <= LSE_MAX, f"{what}: max|dLSE| {dL.max():.3e} > {LSE_MAX}"
    return float(dO.max()), float(dO.mean()), float(dL.max())


class DeviceCache:
    """Host view of a device KV cache [num_blocks, H, block_size, d] that
    copies one physical block (as float64) on access, so the oracle can
    resolve a block table against a large device pool."""

    def __init__(self, t):
        self.t = t
        self.shape = tuple(t.shape)

    def __getitem__(self, i):
        return self.t[int(i)].double().cpu().numpy()
