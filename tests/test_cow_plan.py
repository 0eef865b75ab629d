"""Copy-on-write for the paged KV cache: the host planner and the whole step.

paged_cow_plan (the library's host helper, C ABI) decides which pending
writes hit a block shared by several sequences, takes free blocks for them,
redirects the writers' table entries and adjusts the reference counts
("一文掌握大模型推理加速：FlashAttention与PagedAttention技术详解", section 三
内存共享机制).  On the CPU it is checked against the oracle's restatement
(oracle.cow_plan, itself pinned in test_oracle.py) on random shared-prefix
batches: the same table, counts, free list and copy pairs, exactly; errors
leave every array as it was.  On the GPU the whole step runs: plan ->
paged_block_copy -> paged_kv_append -> paged_attn_decode, against the
oracle's plan -> block_copy -> kv_append -> paged_decode.
"""
import numpy as np
import pytest
import torch

import oracle
from tests._parity import check_close


def _osp():
    import online_softmax_paged_b200 as osp
    osp.load()
    return osp


def _state(rng, S, mb, nb, groups, prefix_blocks):
    """A table whose groups of sequences share their first prefix_blocks
    blocks, the counts of that table, and the unused blocks as free list."""
    pool = [int(b) for b in rng.permutation(nb)]
    table = np.full((S, mb), -1, dtype=np.int32)
    shared = {g: [pool.pop() for _ in range(prefix_blocks)] for g in range(groups)}
    lens = np.zeros(S, dtype=np.int32)
    for s in range(S):
        n = int(rng.integers(1, mb))  # blocks in use; one entry left for an append
        for lb in range(n):
            table[s, lb] = shared[s % groups][lb] if lb < prefix_blocks else pool.pop()
        lens[s] = n
    refs = np.zeros(nb, dtype=np.int32)
    for b in table[table >= 0]:
        refs[b] += 1
    return table, refs, np.array(pool, dtype=np.int32), lens


@pytest.mark.parametrize("seed", range(6))
def test_planner_matches_oracle(seed):
    osp = _osp()
    rng = np.random.default_rng(seed)
    table, refs, free, nblk = _state(rng, S=9, mb=6, nb=80, groups=3, prefix_blocks=3)
    live = [(s, lb) for s in range(9) for lb in range(6) if table[s, lb] >= 0]
    writes = [live[i] for i in rng.integers(0, len(live), 15)]
    t_ref, r_ref, f_ref, src_ref, dst_ref = oracle.cow_plan(table, refs, list(free), writes)
    t, r, f = table.copy(), refs.copy(), free.copy()
    ws = np.array([w[0] for w in writes], dtype=np.int32)
    wb = np.array([w[1] for w in writes], dtype=np.int32)
    src, dst, fc = osp.paged_cow_plan(t, r, f, len(f), ws, wb)
    assert src.tolist() == src_ref and dst.tolist() == dst_ref
    np.testing.assert_array_equal(t, t_ref)
    np.testing.assert_array_equal(r, r_ref)
    assert f[:fc].tolist() == f_ref


def test_planner_errors_leave_arrays_unchanged():
    osp = _osp()
    table = np.array([[4, 1], [4, 3], [4, -1]], dtype=np.int32)
    refs = np.array([0, 1, 0, 1, 3, 0, 0, 0, 0, 0], dtype=np.int32)
    free = np.array([9, 7], dtype=np.int32)
    ws = np.array([0, 1, 2], dtype=np.int32)
    wb = np.array([0, 0, 0], dtype=np.int32)
    # one free block for the two copies the batch needs: ATTN_ENOBLOCKS, nothing changed
    t, r, f = table.copy(), refs.copy(), free.copy()
    with pytest.raises(osp.AttnError) as e:
        osp.paged_cow_plan(t, r, f, 1, ws, wb)
    assert e.value.status == osp.ATTN_ENOBLOCKS
    np.testing.assert_array_equal(t, table)
    np.testing.assert_array_equal(r, refs)
    np.testing.assert_array_equal(f, free)
    # with both free blocks it goes through: the third writer owns block 4 by then
    src, dst, fc = osp.paged_cow_plan(t, r, f, 2, ws, wb)
    assert src.tolist() == [4, 4] and dst.tolist() == [7, 9] and fc == 0
    assert t[:, 0].tolist() == [7, 9, 4] and r[4] == 1 and r[7] == 1 and r[9] == 1
    # invalid batches: a write with no block, outside the table, a stale count, a referenced "free" block
    for tb, rc, fl, s_, b_ in [
        (table, refs, free, [2], [1]),
        (table, refs, free, [3], [0]),
        (table, np.where(np.arange(10) == 1, 0, refs).astype(np.int32), free, [0], [1]),
        (table, refs, np.array([3], dtype=np.int32), [0], [0]),
    ]:
        t, r, f = tb.copy(), rc.copy(), fl.copy()
        with pytest.raises(osp.AttnError) as e:
            osp.paged_cow_plan(t, r, f, len(f), np.array(s_, dtype=np.int32), np.array(b_, dtype=np.int32))
        assert e.value.status == 1  # ATTN_EINVAL
        np.testing.assert_array_equal(t, tb)
        np.testing.assert_array_equal(r, rc)
        np.testing.assert_array_equal(f, fl)
    # an empty batch plans nothing
    src, dst, fc = osp.paged_cow_plan(table.copy(), refs.copy(), free.copy(), 2, np.zeros(0, np.int32),
                                      np.zeros(0, np.int32))
    assert src.size == 0 and dst.size == 0 and fc == 2


@pytest.mark.gpu
def test_copy_on_write_append_then_decode():
    """Sequences of three groups share their first two 16-token blocks; each
    appends one token at position L_s, so the writers whose last block is a
    shared one need a copy first.  The library's step (plan, block copy,
    append, decode) equals the oracle's: the caches bit for bit, the decode
    within the bf16 tolerance; the plan is the oracle's exactly."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    osp = _osp()
    rng = np.random.default_rng(5)
    S, mb, nb, bs, H, d = 12, 6, 200, 16, 4, 128
    table, refs, free, nblk = _state(rng, S=S, mb=mb, nb=nb, groups=3, prefix_blocks=2)
    # lengths end inside each sequence's last block (shared prefix blocks are full
    # for a sequence that has more blocks); the append goes to position L
    lens = np.array([int((n - 1) * bs + rng.integers(1, bs)) for n in nblk], dtype=np.int32)
    writes = [(s, int(lens[s]) // bs) for s in range(S)]
    t_ref, r_ref, f_ref, src_ref, dst_ref = oracle.cow_plan(table, refs, list(free), writes)
    assert len(src_ref) > 0  # the batch does exercise copies
    t, r, f = table.copy(), refs.copy(), free.copy()
    src, dst, fc = osp.paged_cow_plan(t, r, f, len(f), np.array([w[0] for w in writes], dtype=np.int32),
                                      np.array([w[1] for w in writes], dtype=np.int32))
    assert src.tolist() == src_ref and dst.tolist() == dst_ref
    np.testing.assert_array_equal(t, t_ref)

    g = torch.Generator().manual_seed(6)
    kc = torch.randn((nb, H, bs, d), generator=g).to(torch.bfloat16)
    vc = torch.randn((nb, H, bs, d), generator=g).to(torch.bfloat16)
    k_new = torch.randn((S, H, d), generator=g).to(torch.bfloat16)
    v_new = torch.randn((S, H, d), generator=g).to(torch.bfloat16)
    q = torch.randn((S, H, d), generator=g).to(torch.bfloat16)
    dev = "cuda"
    kd, vd = kc.to(dev), vc.to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    osp.paged_block_copy(kd, vd, torch.from_numpy(src).to(dev), torch.from_numpy(dst).to(dev), err_flag=err)
    td = torch.from_numpy(t).to(dev)
    seq_ids = torch.arange(S, dtype=torch.int32, device=dev)
    pos = torch.from_numpy(lens).to(dev)
    osp.paged_kv_append(k_new.to(dev), v_new.to(dev), seq_ids, pos, td, kd, vd, err_flag=err)
    new_lens = torch.from_numpy(lens + 1).to(dev)
    O, LSE = osp.paged_attn_decode(q.to(dev), kd, vd, td, new_lens, bs, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0

    k64, v64 = kc.double().numpy(), vc.double().numpy()
    k2, v2, skipped = oracle.block_copy(k64, v64, src_ref, dst_ref)
    assert skipped == []
    k3, v3, skipped = oracle.kv_append(k2, v2, t_ref, k_new.double().numpy(), v_new.double().numpy(),
                                       np.arange(S), lens, bs)
    assert skipped == []
    # the caches: copies and writes are exact
    np.testing.assert_array_equal(kd.double().cpu().numpy(), k3)
    np.testing.assert_array_equal(vd.double().cpu().numpy(), v3)
    # the sharers that did not copy still read the old prefix blocks
    O_ref, L_ref = oracle.paged_decode(q.double().numpy(), k3, v3, t_ref, lens + 1, bs, 1.0 / np.sqrt(d))
    check_close(O, LSE, O_ref, L_ref, torch.bfloat16, "copy-on-write append + decode")


def _random_state(data_seed):
    """A random, mostly consistent block pool: shared and private blocks in a
    table, the counts of its references, the unused blocks as a shuffled free
    list (sometimes cut short), and a batch of writes that are mostly to
    entries holding a block, sometimes outside the table or to empty entries."""
    rng = np.random.default_rng(data_seed)
    S, mb, nb = int(rng.integers(1, 7)), int(rng.integers(1, 6)), int(rng.integers(4, 41))
    table = np.full((S, mb), -1, dtype=np.int32)
    pool = [int(b) for b in rng.permutation(nb)]
    shared = [pool.pop() for _ in range(int(rng.integers(0, min(4, len(pool)) + 1)))]
    for s in range(S):
        for lb in range(int(rng.integers(0, mb + 1))):
            if shared and rng.random() < 0.5:
                table[s, lb] = shared[int(rng.integers(0, len(shared)))]
            elif pool:
                table[s, lb] = pool.pop()
    refs = np.zeros(nb, dtype=np.int32)
    for b in table[table >= 0]:
        refs[b] += 1
    free = np.array(pool[:int(rng.integers(0, len(pool) + 1))], dtype=np.int32)
    live = [(s, lb) for s in range(S) for lb in range(mb) if table[s, lb] >= 0]
    writes = []
    for _ in range(int(rng.integers(0, 12))):
        u = rng.random()
        if live and u < 0.9:
            writes.append(live[int(rng.integers(0, len(live)))])
        else:
            writes.append((int(rng.integers(-1, S + 1)), int(rng.integers(-1, mb + 1))))
    return table, refs, free, writes


@pytest.mark.parametrize("seed", range(200))
def test_planner_random_batches_match_oracle(seed):
    """Random pools and batches, some of them invalid or short of free
    blocks: the library succeeds exactly when the oracle does, with the same
    table, counts, free list and copy pairs; when it fails it leaves every
    array as it was (all or nothing), and a batch whose writes are all valid
    but which runs out of free blocks reports ATTN_ENOBLOCKS."""
    osp = _osp()
    table, refs, free, writes = _random_state(1000 + seed)
    try:
        expect = oracle.cow_plan(table, refs, list(free), writes)
        err = None
    except ValueError as e:
        expect, err = None, str(e)
    t, r, f = table.copy(), refs.copy(), free.copy()
    ws = np.array([w[0] for w in writes], dtype=np.int32)
    wb = np.array([w[1] for w in writes], dtype=np.int32)
    if expect is not None:
        src, dst, fc = osp.paged_cow_plan(t, r, f, len(f), ws, wb)
        t_ref, r_ref, f_ref, src_ref, dst_ref = expect
        assert src.tolist() == src_ref and dst.tolist() == dst_ref
        np.testing.assert_array_equal(t, t_ref)
        np.testing.assert_array_equal(r, r_ref)
        assert f[:fc].tolist() == f_ref
    else:
        with pytest.raises(osp.AttnError) as e:
            osp.paged_cow_plan(t, r, f, len(f), ws, wb)
        np.testing.assert_array_equal(t, table)
        np.testing.assert_array_equal(r, refs)
        np.testing.assert_array_equal(f, free)
        S, mb = table.shape
        all_valid = all(0 <= s < S and 0 <= lb < mb and table[s, lb] >= 0 for s, lb in writes)
        if all_valid and "ran out" in err:
            assert e.value.status == osp.ATTN_ENOBLOCKS
        else:
            assert e.value.status in (1, osp.ATTN_ENOBLOCKS)
