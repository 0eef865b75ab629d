"""GPU parity of the KV-cache writes (paged_kv_append, paged_block_copy)
against the oracle: both are copies, so the caches must match bit for bit;
end to end, appended and copied-on-write caches must decode to the dense
attention oracle."""
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


def _to_dtype(x, like):
    return torch.from_numpy(np.ascontiguousarray(x)).to(like.dtype).to(like.device)


@pytest.mark.parametrize("dtype,d,bs", [(torch.bfloat16, 128, 16), (torch.bfloat16, 64, 32),
                                        (torch.float32, 128, 32), (torch.float32, 64, 16)])
def test_append_bit_exact(dtype, d, bs):
    osp = _osp()
    g = torch.Generator(device="cuda").manual_seed(3)
    H, nb, S, mb = 4, 200, 6, 9
    kc = torch.randn((nb, H, bs, d), generator=g, device="cuda").to(dtype)
    vc = torch.randn((nb, H, bs, d), generator=g, device="cuda").to(dtype)
    table = torch.randperm(nb, generator=g, device="cuda")[:S * mb].view(S, mb).to(torch.int32).contiguous()
    T = 300
    seq_ids = torch.randint(0, S, (T,), generator=g, device="cuda", dtype=torch.int32)
    # distinct (sequence, position) pairs so the result is unique
    flat = torch.randperm(S * mb * bs, generator=g, device="cuda")[:T]
    seq_ids = (flat // (mb * bs)).to(torch.int32)
    pos = (flat % (mb * bs)).to(torch.int32)
    kn = torch.randn((T, H, d), generator=g, device="cuda").to(dtype)
    vn = torch.randn((T, H, d), generator=g, device="cuda").to(dtype)
    k_ref, v_ref, skipped = oracle.kv_append(to64(kc), to64(vc), table.cpu().numpy(), to64(kn), to64(vn),
                                             seq_ids.cpu().numpy(), pos.cpu().numpy(), bs)
    assert skipped == []
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    osp.paged_kv_append(kn, vn, seq_ids, pos, table, kc, vc, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(kc, _to_dtype(k_ref, kc)) and torch.equal(vc, _to_dtype(v_ref, vc))


def test_append_out_of_range_skipped_and_flagged():
    osp = _osp()
    H, nb, bs, d = 2, 20, 16, 128
    kc = torch.zeros((nb, H, bs, d), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    table = torch.tensor([[3, 25], [4, 5]], dtype=torch.int32, device="cuda")  # 25 is outside the pool
    seq_ids = torch.tensor([0, 0, 2, 1, -1, 1], dtype=torch.int32, device="cuda")
    pos = torch.tensor([1, 20, 0, 40, 0, 17], dtype=torch.int32, device="cuda")
    kn = torch.ones((6, H, d), dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    osp.paged_kv_append(kn, kn, seq_ids, pos, table, kc, vc, err_flag=err)
    bits = osp.attn_read_error(err)
    assert bits & osp.ATTN_DEVERR_BLOCK_TABLE and bits & osp.ATTN_DEVERR_INDEX
    k_ref, _, skipped = oracle.kv_append(to64(torch.zeros_like(kc)), to64(torch.zeros_like(kc)),
                                         table.cpu().numpy(), to64(kn), to64(kn), seq_ids.cpu().numpy(),
                                         pos.cpu().numpy(), bs)
    assert skipped == [1, 2, 3, 4]
    assert torch.equal(kc, _to_dtype(k_ref, kc))


def test_append_then_decode_matches_dense():
    """Fill two sequences through paged_kv_append (random physical blocks),
    then decode: equals the dense oracle on the contiguous K/V."""
    osp = _osp()
    H, d, bs, nb = 8, 128, 16, 300
    lens = [700, 333]
    g = torch.Generator(device="cuda").manual_seed(5)
    kc = torch.zeros((nb, H, bs, d), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    mb = -(-max(lens) // bs)
    perm = torch.randperm(nb, generator=g, device="cuda").to(torch.int32)
    table = torch.full((2, mb), -1, dtype=torch.int32, device="cuda")
    table[0, :-(-lens[0] // bs)] = perm[:-(-lens[0] // bs)]
    table[1, :-(-lens[1] // bs)] = perm[100:100 + -(-lens[1] // bs)]
    Ks = [torch.randn((L, H, d), generator=g, device="cuda").to(torch.bfloat16) for L in lens]
    Vs = [torch.randn((L, H, d), generator=g, device="cuda").to(torch.bfloat16) for L in lens]
    for s, L in enumerate(lens):
        sid = torch.full((L,), s, dtype=torch.int32, device="cuda")
        pos = torch.arange(L, dtype=torch.int32, device="cuda")
        osp.paged_kv_append(Ks[s], Vs[s], sid, pos, table, kc, vc)
    q = torch.randn((2, H, d), generator=g, device="cuda").to(torch.bfloat16)
    sl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    O, LSE = osp.paged_attn_decode(q, kc, vc, table, sl, bs)
    torch.cuda.synchronize()
    for s, L in enumerate(lens):
        for h in range(H):
            o, lse = oracle.attention_head(to64(q[s, h:h + 1]), to64(Ks[s][:, h]), to64(Vs[s][:, h]), False,
                                           d ** -0.5)
            check_close(O[s, h:h + 1], LSE[s, h:h + 1], o, lse, torch.bfloat16, f"append+decode s={s} h={h}")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_block_copy_bit_exact(dtype):
    osp = _osp()
    g = torch.Generator(device="cuda").manual_seed(7)
    nb, H, bs, d = 64, 4, 32, 128
    kc = torch.randn((nb, H, bs, d), generator=g, device="cuda").to(dtype)
    vc = torch.randn((nb, H, bs, d), generator=g, device="cuda").to(dtype)
    perm = torch.randperm(nb, generator=g, device="cuda").to(torch.int32)
    src, dst = perm[:20].contiguous(), perm[20:40].contiguous()
    k_ref, v_ref, skipped = oracle.block_copy(to64(kc), to64(vc), src.cpu().numpy(), dst.cpu().numpy())
    assert skipped == []
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    osp.paged_block_copy(kc, vc, src, dst, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(kc, _to_dtype(k_ref, kc)) and torch.equal(vc, _to_dtype(v_ref, vc))


def test_block_copy_bad_ids_skipped():
    osp = _osp()
    kc = torch.randn((10, 2, 16, 64), device="cuda").to(torch.bfloat16)
    vc = torch.randn((10, 2, 16, 64), device="cuda").to(torch.bfloat16)
    k0, v0 = kc.clone(), vc.clone()
    src = torch.tensor([1, 12, 3], dtype=torch.int32, device="cuda")
    dst = torch.tensor([5, 6, -1], dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    osp.paged_block_copy(kc, vc, src, dst, err_flag=err)
    assert osp.attn_read_error(err) & osp.ATTN_DEVERR_BLOCK_TABLE
    assert torch.equal(kc[5], k0[1]) and torch.equal(vc[5], v0[1])
    keep = [b for b in range(10) if b != 5]
    assert torch.equal(kc[keep], k0[keep]) and torch.equal(vc[keep], v0[keep])


def test_copy_on_write_then_decode():
    """Eight sequences share a 512-token prefix (shared-prefix generator).
    Sequence 3 diverges: its partially filled last prefix block is copied to a
    free block, its table entry redirected and one new token appended there.
    Every sequence then decodes to its own oracle result (sequence 3 sees the
    new token, the others the original block)."""
    osp = _osp()
    p = W.paged_shared_prefix(num_seqs=8, H=4, d=128, block_size=32, pool=400, median=300, sigma=0.3, len_lo=40,
                              len_hi=1000, group=8, prefix_tokens=512, seed=9, device="cuda")
    sl = p.seq_lens.clone()
    sl[3] = 100  # sequence 3: 100 tokens, its 4th block (tokens 96..127) is shared
    table = p.block_table.clone()
    used = set(table[table >= 0].cpu().tolist())
    free = [b for b in range(p.num_blocks) if b not in used][0]
    lb = 100 // 32
    src = table[3, lb:lb + 1].contiguous()
    dst = torch.tensor([free], dtype=torch.int32, device="cuda")
    osp.paged_block_copy(p.k_cache, p.v_cache, src, dst)
    table[3, lb] = free
    kn = torch.randn((1, 4, 128), device="cuda").to(torch.bfloat16)
    osp.paged_kv_append(kn, kn, torch.tensor([3], dtype=torch.int32, device="cuda"),
                        torch.tensor([100], dtype=torch.int32, device="cuda"), table, p.k_cache, p.v_cache)
    sl[3] = 101
    O, LSE = osp.paged_attn_decode(p.q, p.k_cache, p.v_cache, table, sl, 32, scale=p.scale)
    torch.cuda.synchronize()

    class Dev:
        def __init__(self, t):
            self.t, self.shape = t, tuple(t.shape)

        def __getitem__(self, i):
            return self.t[int(i)].float().cpu().numpy()

    O_ref, L_ref = oracle.paged_decode(to64(p.q), Dev(p.k_cache), Dev(p.v_cache), table.cpu().numpy(),
                                       sl.cpu().numpy(), 32, p.scale)
    check_close(O, LSE, O_ref, L_ref, torch.bfloat16, "copy-on-write + decode")
    # the shared block itself is untouched: another sequence that still uses it sees the old slot 4
    other = [s for s in range(8) if s != 3 and int(sl[s]) > 100 and int(table[s, lb]) == int(src[0])]
    if other:
        assert not torch.equal(p.k_cache[int(src[0]), :, 100 % 32], kn[0])
