"""GPU parity of multi-token paged prefill (paged_attn_prefill) against the
fp64 oracle.

Each sequence holds L_s cached tokens of which the last n_s are new; new
token i sits at position L_s - n_s + i and attends keys 0 .. that position
through the block table.  Small mixes are checked in full (pure prefill,
chunks after a context, one-token chunks, empty chunks, lengths that end
inside a block and inside a 16-key step, multi-head and grouped heads,
block sizes 16/32, d 64/128); the chunked-prefill workload on sampled rows.
Physical placement shuffles must give bit-identical output, NaN in unused
cache slots must not leak into any row, and bad tables, lengths and offsets
set the device error bits.
"""
import numpy as np
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
    import online_softmax_paged_b200 as osp
    osp.load()


def _osp():
    import online_softmax_paged_b200 as osp
    return osp


def _run(p, err=None, **kw):
    O, LSE = _osp().paged_attn_prefill(p.q, p.k_cache, p.v_cache, p.block_table, p.seq_lens, p.cu_q,
                                       p.block_size, scale=p.scale, err_flag=err, **kw)
    torch.cuda.synchronize()
    return O, LSE


def _oracle(p, seqs=None):
    return oracle.paged_prefill(to64(p.q), DeviceCache(p.k_cache), DeviceCache(p.v_cache),
                                p.block_table.cpu().numpy(), p.seq_lens.cpu().numpy(), p.cu_q.cpu().numpy(),
                                p.block_size, p.scale, seqs=seqs)


def _rows(cu, seqs):
    return [r for s in seqs for r in range(int(cu[s]), int(cu[s + 1]))]


# (cached context, new tokens) per sequence: pure prefills of 1, 5, 257 and
# 300 tokens; chunks after a context (17 after 983, 256 after 444, 513 after
# 87); one new token (decode) after 2047; an empty chunk; 128 after 1.
MIX = [(0, 1), (0, 5), (0, 300), (983, 17), (444, 256), (87, 513), (2047, 1), (50, 0), (1, 128), (0, 257)]


@pytest.mark.parametrize("Hq,Hkv,d,bs", [(8, 8, 128, 16), (8, 2, 128, 32), (8, 8, 64, 32), (8, 1, 64, 16),
                                         (4, 2, 128, 16)])
def test_mix_full(Hq, Hkv, d, bs):
    ctx, n = zip(*MIX)
    p = W.paged_prefill_inputs(ctx, n, Hq=Hq, Hkv=Hkv, d=d, block_size=bs, seed=Hq + Hkv + d + bs, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O, LSE = _run(p, err)
    assert int(err.item()) == 0
    O_ref, L_ref = _oracle(p)
    check_close(O, LSE, O_ref, L_ref, torch.bfloat16, f"paged prefill Hq={Hq} Hkv={Hkv} d={d} bs={bs}")


def test_placement_shuffle_bit_identical():
    ctx, n = zip(*MIX)
    p = W.paged_prefill_inputs(ctx, n, Hq=8, Hkv=2, d=128, block_size=16, seed=5, device="cuda")
    O1, L1 = _run(p)
    for seed in (1, 2):
        O2, L2 = _run(p.shuffled(seed))
        assert torch.equal(O1, O2) and torch.equal(L1, L2)


def test_nan_in_unused_slots_does_not_leak():
    """Every cache slot that no sequence uses (tails of last blocks, unused
    blocks) is NaN: the rows must equal the clean run bit for bit."""
    ctx, n = zip(*MIX)
    p = W.paged_prefill_inputs(ctx, n, Hq=8, Hkv=2, d=128, block_size=32, seed=6, device="cuda")
    O1, L1 = _run(p)
    kc, vc = p.k_cache.clone(), p.v_cache.clone()
    live = torch.zeros(kc.shape[0], kc.shape[2], dtype=torch.bool)
    t, sl = p.block_table.cpu(), p.seq_lens.cpu()
    for s in range(t.shape[0]):
        L = int(sl[s])
        for lb in range(-(-L // p.block_size)):
            live[int(t[s, lb]), :min(p.block_size, L - lb * p.block_size)] = True
    dead = (~live).to("cuda")
    kc.masked_fill_(dead[:, None, :, None], float("nan"))
    vc.masked_fill_(dead[:, None, :, None], float("nan"))
    q = W.PagedPrefillInputs(p.q, kc, vc, p.block_table, p.seq_lens, p.cu_q, p.block_size, p.scale)
    O2, L2 = _run(q)
    assert torch.isfinite(O2.float()).all()
    assert torch.equal(O1, O2) and torch.equal(L1, L2)


def test_pure_prefill_matches_dense_causal():
    """Paging changes storage, not the math: a sequence whose every token is
    new gives (within tolerance of the same oracle) the dense causal prefill."""
    osp = _osp()
    H, d, bs, N = 4, 128, 16, 777
    p = W.paged_prefill_inputs([0], [N], Hq=H, Hkv=H, d=d, block_size=bs, seed=8, device="cuda")
    O, LSE = _run(p)
    nb = -(-N // bs)
    t = p.block_table[0, :nb].long()
    K = p.k_cache[t].permute(1, 0, 2, 3).reshape(H, nb * bs, d)[:, :N].unsqueeze(0).contiguous()
    V = p.v_cache[t].permute(1, 0, 2, 3).reshape(H, nb * bs, d)[:, :N].unsqueeze(0).contiguous()
    Q = p.q.permute(1, 0, 2).unsqueeze(0).contiguous()
    Od, Ld = osp.attn_fwd(Q, K, V, causal=True)
    torch.cuda.synchronize()
    assert (O.permute(1, 0, 2).float() - Od[0].float()).abs().max().item() <= 2e-2
    assert (LSE.t() - Ld[0]).abs().max().item() <= 1e-3


def test_chunked_prefill_workload_sampled():
    """The chunked-prefill workload (8 sequences, 2048 new tokens after
    U{0..6144} cached, 32 query heads over 8 key/value heads, bs 16): 24 rows
    (first, last, 22 random) of each of 6 (sequence, head) pairs against the
    oracle; all rows finite; a placement shuffle is bit-identical."""
    p = W.paged_chunked_prefill(device="cuda", seed=0, **{k: v for k, v in W.PREFILL_PAGED_CHUNKED.items()})
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O, LSE = _run(p, err)
    assert int(err.item()) == 0
    assert torch.isfinite(O.float()).all() and torch.isfinite(LSE).all()
    cu, sl = p.cu_q.cpu().numpy(), p.seq_lens.cpu().numpy()
    G = p.q.shape[1] // p.k_cache.shape[1]
    rng = np.random.default_rng(0)
    kd, vd = DeviceCache(p.k_cache), DeviceCache(p.v_cache)
    for s, h in [(0, 0), (3, 31), (7, 9), (int(sl.argmax()), 17), (int(sl.argmin()), 4), (5, 26)]:
        L, n = int(sl[s]), int(cu[s + 1] - cu[s])
        Ks = oracle.gather_paged(kd, p.block_table[s].cpu().numpy(), L, p.block_size)[h // G]
        Vs = oracle.gather_paged(vd, p.block_table[s].cpu().numpy(), L, p.block_size)[h // G]
        rows = sorted({0, n - 1, *rng.integers(0, n, 22).tolist()})
        o_ref, l_ref = [], []
        for i in rows:
            pos = L - n + i
            o, l = oracle.attention_head(to64(p.q[cu[s] + i, h:h + 1]), Ks[:pos + 1], Vs[:pos + 1], False, p.scale)
            o_ref.append(o[0])
            l_ref.append(l[0])
        idx = [int(cu[s]) + i for i in rows]
        check_close(O[idx, h], LSE[idx, h], np.array(o_ref), np.array(l_ref), torch.bfloat16,
                    f"chunked prefill s={s} h={h}")
    O2, L2 = _run(p.shuffled(4))
    assert torch.equal(O, O2) and torch.equal(LSE, L2)


def test_bad_table_entry_flagged():
    osp = _osp()
    p = W.paged_prefill_inputs([100, 0, 40], [20, 33, 7], Hq=4, Hkv=4, d=128, block_size=16, seed=9, device="cuda")
    t = p.block_table.clone()
    t[0, 2] = p.k_cache.shape[0] + 3
    bad = W.PagedPrefillInputs(p.q, p.k_cache, p.v_cache, t, p.seq_lens, p.cu_q, p.block_size, p.scale)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    O, LSE = _run(bad, err)
    assert osp.attn_read_error(err) & osp.ATTN_DEVERR_BLOCK_TABLE
    good = [1, 2]
    rows = _rows(p.cu_q.cpu(), good)
    O_ref, L_ref = _oracle(p, seqs=good)
    check_close(O[rows], LSE[rows], O_ref[rows], L_ref[rows], torch.bfloat16, "rows beside a bad table entry")


def test_bad_lengths_and_offsets_flagged_rows_untouched():
    osp = _osp()
    p = W.paged_prefill_inputs([10, 0, 300, 5], [20, 33, 7, 9], Hq=4, Hkv=2, d=64, block_size=32, seed=10,
                               device="cuda")
    sl = p.seq_lens.clone()
    sl[1] = 32       # 33 new tokens but 32 cached: SEQ_LEN
    sl[2] = p.block_table.shape[1] * 32 + 1  # more keys than the table holds: SEQ_LEN
    bad = W.PagedPrefillInputs(p.q, p.k_cache, p.v_cache, p.block_table, sl, p.cu_q, p.block_size, p.scale)
    O = torch.full_like(p.q, 7.0)
    LSE = torch.full(p.q.shape[:2], 7.0, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    _run(bad, err, O=O, LSE=LSE)
    assert osp.attn_read_error(err) & osp.ATTN_DEVERR_SEQ_LEN
    cu = p.cu_q.cpu()
    for s in (1, 2):
        r = _rows(cu, [s])
        assert (O[r] == 7.0).all() and (LSE[r] == 7.0).all()
    good = [0, 3]
    O_ref, L_ref = _oracle(p, seqs=good)
    r = _rows(cu, good)
    check_close(O[r], LSE[r], O_ref[r], L_ref[r], torch.bfloat16, "rows beside bad lengths")
    # cu_q past total_q: INDEX, that sequence untouched
    cq = p.cu_q.clone()
    cq[4] = cq[4] + 5
    bad2 = W.PagedPrefillInputs(p.q, p.k_cache, p.v_cache, p.block_table, p.seq_lens, cq, p.block_size, p.scale)
    O.fill_(7.0)
    err.zero_()
    _run(bad2, err, O=O, LSE=LSE, max_q_per_seq=64)
    assert osp.attn_read_error(err) & osp.ATTN_DEVERR_INDEX
    assert (O[_rows(cu, [3])] == 7.0).all()


def test_host_validation():
    osp = _osp()
    p = W.paged_prefill_inputs([0], [10], Hq=6, Hkv=4, d=128, block_size=16, seed=11, device="cuda")
    with pytest.raises(osp.AttnError):  # 6 query heads over 4 key/value heads
        _run(p)
    p = W.paged_prefill_inputs([0], [10], Hq=4, Hkv=4, d=96, block_size=16, seed=11, device="cuda")
    with pytest.raises(osp.AttnError):  # d = 96
        _run(p)


def test_empty_batch_is_a_no_op():
    p = W.paged_prefill_inputs([5, 9], [0, 0], Hq=4, Hkv=4, d=128, block_size=16, seed=12, device="cuda")
    O, LSE = _run(p)
    assert O.shape == (0, 4, 128) and LSE.shape == (0, 4)
