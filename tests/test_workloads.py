"""Host-side checks of the seeded input generators (no GPU)."""
import numpy as np
import torch

import oracle
import workloads as W


def test_dense_inputs_seeded_and_rounded():
    a = W.dense_inputs(1, 2, 33, 8, dtype=torch.bfloat16, seed=3)
    b = W.dense_inputs(1, 2, 33, 8, dtype=torch.bfloat16, seed=3)
    for k in ("Q", "K", "V"):
        assert a[k].dtype == torch.bfloat16 and a[k].shape == (1, 2, 33, 8)
        assert torch.equal(a[k], b[k])
    assert not torch.equal(a["Q"], a["K"])
    assert abs(a["scale"] - 1 / np.sqrt(8)) < 1e-15
    half = W.dense_inputs(1, 2, 33, 8, dtype=torch.float32, mult=0.5, seed=3)
    full = W.dense_inputs(1, 2, 33, 8, dtype=torch.float32, mult=1.0, seed=3)
    assert torch.equal(half["Q"] * 2, full["Q"])


def test_paged_uniform_table_without_replacement():
    p = W.paged_uniform(num_seqs=16, H=2, d=8, block_size=16, pool=600, len_lo=1, len_hi=300, seed=0)
    t = p.block_table.numpy()
    sl = p.seq_lens.numpy()
    assert ((sl >= 1) & (sl <= 300)).all()
    used = []
    for s in range(16):
        nb = -(-int(sl[s]) // 16)
        assert (t[s, :nb] >= 0).all() and (t[s, :nb] < 600).all()
        assert (t[s, nb:] == -1).all()
        used.extend(t[s, :nb].tolist())
    assert len(used) == len(set(used)), "a physical block appears twice"
    assert p.max_blocks_per_seq == -(-300 // 16)


def test_paged_shared_prefix_groups():
    p = W.paged_shared_prefix(num_seqs=24, H=2, d=8, block_size=32, pool=2000, median=300, sigma=1.0,
                              len_lo=1, len_hi=1024, group=8, prefix_tokens=128, seed=0)
    t = p.block_table.numpy()
    sl = p.seq_lens.numpy()
    assert ((sl >= 1) & (sl <= 1024)).all()
    pb = 128 // 32
    owner = {}
    for members in p.shared_groups:
        longest = max(members, key=lambda s: sl[s])
        prefix = t[longest, :pb]
        for s in members:
            nb = -(-int(sl[s]) // 32)
            n_shared = min(nb, -(-min(int(sl[s]), 128) // 32))
            assert (t[s, :n_shared] == prefix[:n_shared]).all()
            for lb in range(n_shared, nb):
                phys = int(t[s, lb])
                assert phys not in owner, "private block reused"
                owner[phys] = s
            assert (t[s, nb:] == -1).all()
    shared_ids = set(t[:, :pb].ravel().tolist()) - {-1}
    assert not (shared_ids & set(owner)), "prefix block also used privately"


def test_shuffle_keeps_logical_data():
    p = W.paged_uniform(num_seqs=5, H=2, d=4, block_size=4, pool=80, len_lo=1, len_hi=40, seed=2)
    p2 = W.shuffle_placement(p, seed=7)
    assert not torch.equal(p.block_table, p2.block_table)
    for s in range(5):
        L = int(p.seq_lens[s])
        a = oracle.gather_paged(p.k_cache.float().numpy(), p.block_table[s].numpy(), L, 4)
        b = oracle.gather_paged(p2.k_cache.float().numpy(), p2.block_table[s].numpy(), L, 4)
        np.testing.assert_array_equal(a, b)


def test_byte_counts():
    p = W.paged_shared_prefix(num_seqs=16, H=2, d=8, block_size=32, pool=2000, median=300, sigma=1.0,
                              len_lo=1, len_hi=1024, group=8, prefix_tokens=128, seed=1)
    logical = W.logical_kv_bytes(p)
    unique = W.unique_kv_bytes(p)
    assert logical == int(p.seq_lens.sum()) * 2 * 2 * 8 * 2
    assert unique < logical
    u = W.paged_uniform(num_seqs=6, H=2, d=8, block_size=16, pool=200, len_lo=1, len_hi=100, seed=1)
    assert W.unique_kv_bytes(u) == W.logical_kv_bytes(u)
