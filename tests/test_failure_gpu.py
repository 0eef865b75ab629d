"""The failure path of the bounded pipeline waits, on the GPU.

Every kernel's mbarrier waits give up after a wall-clock limit (1 s),
report ATTN_DEVERR_TIMEOUT in the caller's error word and unwind.  The
library's self-test makes exactly that wait run out -- on a barrier phase
that nothing completes -- without any fault, trap or unbounded spin; the
test checks the reported status and that the context is still usable.
"""
import time

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


def test_wait_limit_reports_timeout_and_context_survives():
    import online_softmax_paged_b200 as osp
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    result = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    osp.attn_selftest_wait_timeout(err, result)
    bits = osp.attn_read_error(err)
    elapsed = time.perf_counter() - t0
    assert bits == osp.ATTN_DEVERR_TIMEOUT, bits
    assert int(result.item()) == 0  # the wait gave up
    assert 0.9 < elapsed < 30.0, elapsed  # the 1 s limit, then a normal return
    # the context still runs the library's kernels correctly
    inp = W.dense_inputs(1, 2, 200, 128, dtype=torch.bfloat16, seed=3, device="cuda", causal=True)
    err2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    O, LSE = osp.attn_fwd(inp["Q"], inp["K"], inp["V"], causal=True, scale=inp["scale"], err_flag=err2)
    assert osp.attn_read_error(err2) == 0
    O_ref, L_ref = oracle.attention_dense(to64(inp["Q"]), to64(inp["K"]), to64(inp["V"]), True, inp["scale"])
    check_close(O, LSE, O_ref, L_ref, torch.bfloat16, "attn_fwd after a timed-out wait")


def test_selftest_rejects_missing_flag():
    import online_softmax_paged_b200 as osp
    assert osp.load().attn_selftest_wait_timeout(None, None, None) == osp.ATTN_EINVAL
