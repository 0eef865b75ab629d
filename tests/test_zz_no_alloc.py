"""paged_attn_decode_noalloc: the decode entry point for callers that cannot
allocate device memory (code running inside an allocator or pool callback,
processes whose device memory is fixed up front, plain C hosts with no
framework to borrow memory from).  It takes no workspace and uses a fixed
scratch array compiled into the library instead.

Checked through the C ABI against the workspace-taking entry point on two
calls in a row with different inputs (the second call runs on whatever the
first left in the shared scratch).  Both entry points run the same plan and
kernels on the same sizes, so O and LSE must be bit-identical, not merely
close; each call is also compared with the oracle on sampled sequences.
Sizes too large for the scratch are refused.  This file is named to be
collected last.
"""
import pytest
import torch

import oracle
import workloads as W
from tests._parity import DeviceCache, check_close, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _both(osp, p):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O_ref, L_ref = osp.paged_attn_decode(p.q, p.k_cache, p.v_cache, p.block_table, p.seq_lens, p.block_size,
                                         scale=p.scale)
    O, L = osp.paged_attn_decode_noalloc(p.q, p.k_cache, p.v_cache, p.block_table, p.seq_lens, p.block_size,
                                         scale=p.scale, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return O, L, O_ref, L_ref


def test_noalloc_matches_workspace_entry_two_calls_in_a_row():
    import online_softmax_paged_b200 as osp
    first = W.paged_uniform(num_seqs=64, H=32, d=128, block_size=16, pool=20000, len_lo=128, len_hi=4096, seed=0,
                            device="cuda")
    second = W.paged_uniform(num_seqs=19, H=8, d=128, block_size=32, pool=3000, len_lo=0, len_hi=3000, seed=5,
                             device="cuda")
    for name, p, seqs in (("first", first, [0, 17, 40, 63]), ("second", second, list(range(19)))):
        O, L, O_ws, L_ws = _both(osp, p)
        # same plan, same kernels, same sizes: identical bits
        assert torch.equal(O, O_ws), f"{name} call: O differs from the workspace entry point"
        assert torch.equal(L, L_ws), f"{name} call: LSE differs from the workspace entry point"
        O_ref, L_ref = oracle.paged_decode(to64(p.q), DeviceCache(p.k_cache), DeviceCache(p.v_cache),
                                           p.block_table.cpu().numpy(), p.seq_lens.cpu().numpy(), p.block_size,
                                           p.scale, seqs=seqs)
        check_close(O[seqs], L[seqs], O_ref[seqs], L_ref[seqs], torch.bfloat16, f"no-alloc vs oracle ({name} call)")


def test_noalloc_refuses_sizes_beyond_scratch():
    import online_softmax_paged_b200 as osp
    S, H, bs, mb = 4096, 64, 32, 1024
    assert osp.paged_attn_decode_workspace_size(S, H, 128, mb, bs) > osp.ATTN_NOALLOC_SCRATCH_BYTES
    q = torch.zeros((S, H, 128), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((1, H, bs, 128), dtype=torch.bfloat16, device="cuda")
    table = torch.zeros((S, mb), dtype=torch.int32, device="cuda")
    lens = torch.ones(S, dtype=torch.int32, device="cuda")
    with pytest.raises(osp.AttnError) as e:
        osp.paged_attn_decode_noalloc(q, kc, kc, table, lens, bs)
    assert e.value.status == 2  # ATTN_EUNSUPPORTED
