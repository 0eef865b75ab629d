"""Pins for the fp64 oracle: checks against things other than the oracle itself.

Each pin is a hand-worked example (tests/golden), a closed form, an
invariant stated by the pages, a library routine that reduces to the same
definition (torch SDPA / logsumexp in fp64), or brute force on tiny inputs.
``test_planted_mistakes_are_caught`` plants plausible errors in copies of the
oracle (on the CPU) and checks that the pins reject every one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as A

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
_NS = {"log": math.log, "exp": math.exp, "e": math.e, "inf": math.inf}


def _ev(x):
    if isinstance(x, list):
        return [_ev(v) for v in x]
    return float(eval(str(x), {"__builtins__": {}}, _NS))  # fixture expressions: numbers, log, exp, e


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# --------------------------------------------------------------------------
# pin functions, parameterised by the implementation so planted mistakes can
# be run through the same checks
# --------------------------------------------------------------------------

def pin_golden_dense(attn):
    g = json.load(open(os.path.join(GOLDEN, "hand_worked_dense.json")))
    Q, K, V = (np.array(_ev(g[k]))[None, None] for k in ("Q", "K", "V"))
    for mode, causal in (("noncausal", False), ("causal", True)):
        O, LSE = attn(Q, K, V, causal, _ev(g["scale"]))
        np.testing.assert_allclose(O[0, 0], np.array(_ev(g[mode]["O"])), rtol=0, atol=1e-13)
        np.testing.assert_allclose(LSE[0, 0], np.array(_ev(g[mode]["LSE"])), rtol=0, atol=1e-13)


def pin_torch_sdpa(attn):
    """Library special case: torch's SDPA in fp64 on the CPU computes the same
    definition; logsumexp of the masked score matrix gives the LSE."""
    for (B, H, N, d), causal in itertools.product([(1, 2, 37, 8), (2, 1, 64, 16)], [False, True]):
        Q, K, V = (_rand((B, H, N, d), s) for s in (1, 2, 3))
        scale = 0.37
        O, LSE = attn(Q, K, V, causal, scale)
        tq, tk, tv = (torch.from_numpy(x) for x in (Q, K, V))
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale)
        np.testing.assert_allclose(O, ref.numpy(), rtol=0, atol=1e-12)
        S = torch.einsum("bhid,bhjd->bhij", tq, tk) * scale
        if causal:
            S = S.masked_fill(torch.triu(torch.ones(N, N, dtype=torch.bool), 1), -math.inf)
        np.testing.assert_allclose(LSE, torch.logsumexp(S, dim=-1).numpy(), rtol=0, atol=1e-12)


def pin_closed_forms(attn):
    B, H, N, d = 1, 2, 19, 4
    V = _rand((B, H, N, d), 7)
    K = _rand((B, H, N, d), 8)
    Z = np.zeros((B, H, N, d))
    # Q = 0: every score is 0 -> LSE = ln(#visible), O = mean of visible V
    O, LSE = attn(Z, K, V, False, 0.5)
    np.testing.assert_allclose(LSE, np.full((B, H, N), math.log(N)), atol=1e-13)
    np.testing.assert_allclose(O, np.broadcast_to(V.mean(axis=2, keepdims=True), O.shape), atol=1e-13)
    O, LSE = attn(Z, K, V, True, 0.5)
    i = np.arange(N)
    np.testing.assert_allclose(LSE, np.broadcast_to(np.log(i + 1.0), LSE.shape), atol=1e-13)
    prefix_mean = np.cumsum(V, axis=2) / (i + 1.0)[None, None, :, None]
    np.testing.assert_allclose(O, prefix_mean, atol=1e-13)
    # causal row 0 attends only key 0: O0 = v0, LSE0 = scale q0.k0
    Q = _rand((B, H, N, d), 9)
    O, LSE = attn(Q, K, V, True, 0.5)
    np.testing.assert_allclose(O[:, :, 0], V[:, :, 0], atol=1e-13)
    np.testing.assert_allclose(LSE[:, :, 0], 0.5 * np.einsum("bhd,bhd->bh", Q[:, :, 0], K[:, :, 0]), atol=1e-13)
    # causal last row equals the non-causal last row
    On, Ln = attn(Q, K, V, False, 0.5)
    np.testing.assert_allclose(O[:, :, -1], On[:, :, -1], atol=1e-13)
    np.testing.assert_allclose(LSE[:, :, -1], Ln[:, :, -1], atol=1e-13)
    # uniform V -> O = v for every row, causal or not
    v = _rand((d,), 10)
    Vu = np.broadcast_to(v, (B, H, N, d)).copy()
    for causal in (False, True):
        O, _ = attn(Q, K, Vu, causal, 0.5)
        np.testing.assert_allclose(O, np.broadcast_to(v, O.shape), atol=1e-13)
    # one key -> O = v0, LSE = scale q.k0
    O, LSE = attn(Q[:, :, :3], K[:, :, :1], V[:, :, :1], False, 0.5)
    np.testing.assert_allclose(O, np.broadcast_to(V[:, :, :1], O.shape), atol=1e-13)
    np.testing.assert_allclose(LSE, 0.5 * np.einsum("bhid,bhd->bhi", Q[:, :, :3], K[:, :, 0]), atol=1e-13)


def _dense(Q, K, V, causal, scale):
    return oracle.attention_dense(Q, K, V, causal, scale)


# --------------------------------------------------------------------------
# the pins applied to the oracle
# --------------------------------------------------------------------------

def test_golden_dense():
    pin_golden_dense(_dense)


def test_torch_sdpa_and_logsumexp():
    pin_torch_sdpa(_dense)


def test_closed_forms():
    pin_closed_forms(_dense)


def test_prob_rows_sum_to_one_and_o_is_pv():
    Q, K, V = (_rand((23, 8), s) for s in (11, 12, 13))
    for causal in (False, True):
        P = A.softmax_probs(Q, K, causal, 0.3)
        np.testing.assert_allclose(P.sum(axis=1), 1.0, atol=1e-14)
        assert (P >= 0).all()
        if causal:
            assert (P[np.triu_indices(23, 1)] == 0).all()
        O, _ = A.attention_head(Q, K, V, causal, 0.3)
        np.testing.assert_allclose(O, P @ V, atol=1e-13)


def test_online_tiled_equals_one_shot_bruteforce():
    """[实现解析] §2.1: the incremental update equals one-shot softmax; every
    tile split of tiny inputs, causal and not."""
    for N, d in [(1, 1), (3, 2), (5, 3), (8, 4)]:
        Q, K, V = (_rand((N, d), 100 + N + s) * 2.0 for s in range(3))
        for causal in (False, True):
            O1, L1 = A.attention_head(Q, K, V, causal, 0.7)
            for Br in range(1, N + 1):
                for Bc in range(1, N + 1):
                    O2, L2 = A.attention_online_tiled(Q, K, V, causal, 0.7, Br, Bc)
                    np.testing.assert_allclose(O2, O1, rtol=0, atol=1e-13)
                    np.testing.assert_allclose(L2, L1, rtol=0, atol=1e-13)


def test_online_tiled_large_score_range():
    # scores spanning ~200 nats: the running max must be subtracted (safe softmax)
    Q, K, V = (_rand((16, 4), s) for s in (21, 22, 23))
    Q *= 30.0
    O1, L1 = A.attention_head(Q, K, V, True, 1.0)
    O2, L2 = A.attention_online_tiled(Q, K, V, True, 1.0, 4, 3)
    assert np.isfinite(O1).all() and np.isfinite(L1).all()
    np.testing.assert_allclose(O2, O1, atol=1e-12)
    np.testing.assert_allclose(L2, L1, rtol=1e-14, atol=1e-11)


def test_invariants_permutation_scaling_shift():
    N, d = 17, 6
    Q, K, V = (_rand((N, d), s) for s in (31, 32, 33))
    O, L = A.attention_head(Q, K, V, False, 0.4)
    perm = np.random.default_rng(5).permutation(N)
    O2, L2 = A.attention_head(Q, K[perm], V[perm], False, 0.4)
    np.testing.assert_allclose(O2, O, atol=1e-13)
    np.testing.assert_allclose(L2, L, atol=1e-13)
    O3, _ = A.attention_head(Q, K, 3.5 * V, False, 0.4)
    np.testing.assert_allclose(O3, 3.5 * O, atol=1e-12)
    # add c to every score: column 0 of Q is 1, key column 0 shifted by c/scale
    Qs = Q.copy()
    Qs[:, 0] = 1.0
    Os, Ls = A.attention_head(Qs, K, V, False, 0.4)
    Ks = K.copy()
    Ks[:, 0] += 2.5 / 0.4
    Os2, Ls2 = A.attention_head(Qs, Ks, V, False, 0.4)
    np.testing.assert_allclose(Os2, Os, atol=1e-12)
    np.testing.assert_allclose(Ls2, Ls + 2.5, atol=1e-12)


def test_brute_c_matches_numpy_dense():
    for causal in (False, True):
        Q, K, V = (_rand((2, 3, 13, 5), s) for s in (41, 42, 43))
        O1, L1 = oracle.attention_dense(Q, K, V, causal, 0.45)
        O2, L2 = oracle.brute_attention(Q, K, V, causal, 0.45)
        np.testing.assert_allclose(O1, O2, atol=1e-13)
        np.testing.assert_allclose(L1, L2, atol=1e-13)


def _tiny_paged(seed=0, S=4, H=2, d=3, bs=4, pool=None, max_blocks=3):
    rng = np.random.default_rng(seed)
    pool = pool or S * max_blocks + 2
    kc = rng.standard_normal((pool, H, bs, d))
    vc = rng.standard_normal((pool, H, bs, d))
    q = rng.standard_normal((S, H, d))
    lens = rng.integers(0, max_blocks * bs + 1, S)
    lens[0] = max_blocks * bs
    perm = rng.permutation(pool)
    table = -np.ones((S, max_blocks), dtype=np.int32)
    cur = 0
    for s in range(S):
        nb = -(-lens[s] // bs)
        table[s, :nb] = perm[cur:cur + nb]
        cur += nb
    return q, kc, vc, table, lens.astype(np.int32), bs


def test_golden_paged():
    g = json.load(open(os.path.join(GOLDEN, "hand_worked_paged.json")))
    q, kc, vc = (np.array(_ev(g[k])) for k in ("q", "k_cache", "v_cache"))
    O, L = oracle.paged_decode(q, kc, vc, np.array(g["block_table"]), np.array(g["seq_lens"]),
                               g["block_size"], _ev(g["scale"]))
    np.testing.assert_allclose(O, np.array(_ev(g["O"])), atol=1e-13)
    np.testing.assert_allclose(L, np.array(_ev(g["LSE"])), atol=1e-13)


def test_paged_python_loops_bruteforce():
    """Pure-python loops, tiny inputs: slot j of sequence s is
    cache[table[s][j // bs], h, j % bs]."""
    q, kc, vc, table, lens, bs = _tiny_paged(1)
    O, L = oracle.paged_decode(q, kc, vc, table, lens, bs, 0.8)
    S, H, d = q.shape
    for s in range(S):
        for h in range(H):
            sc, vs = [], []
            for j in range(int(lens[s])):
                phys = table[s][j // bs]
                k = kc[phys, h, j % bs]
                sc.append(0.8 * sum(q[s, h, c] * k[c] for c in range(d)))
                vs.append(vc[phys, h, j % bs])
            if not sc:
                assert L[s, h] == -math.inf and (O[s, h] == 0).all()
                continue
            m = max(sc)
            w = [math.exp(x - m) for x in sc]
            tot = sum(w)
            for c in range(d):
                assert abs(O[s, h, c] - sum(wi * v[c] for wi, v in zip(w, vs)) / tot) < 1e-13
            assert abs(L[s, h] - (m + math.log(tot))) < 1e-13


def test_brute_c_matches_numpy_paged():
    q, kc, vc, table, lens, bs = _tiny_paged(2, S=6)
    O1, L1 = oracle.paged_decode(q, kc, vc, table, lens, bs, 0.6)
    O2, L2 = oracle.brute_paged_decode(q, kc, vc, table, lens, bs, 0.6)
    np.testing.assert_allclose(O1, O2, atol=1e-13)
    np.testing.assert_allclose(L1, L2, atol=1e-13)


def test_paged_identity_table_equals_dense():
    """[区别] Q2: paging changes storage, not the math.  Block i of a
    sequence at physical i: the decode equals the dense oracle on the last
    query row with a contiguous K/V."""
    H, d, bs, nb = 2, 5, 4, 3
    L = 11
    rng = np.random.default_rng(3)
    K = rng.standard_normal((H, nb * bs, d))
    V = rng.standard_normal((H, nb * bs, d))
    q = rng.standard_normal((1, H, d))
    kc = K.reshape(H, nb, bs, d).transpose(1, 0, 2, 3)
    vc = V.reshape(H, nb, bs, d).transpose(1, 0, 2, 3)
    O, LSE = oracle.paged_decode(q, kc, vc, np.arange(nb)[None], np.array([L]), bs, 0.5)
    for h in range(H):
        o, lse = A.attention_head(q[0, h:h + 1], K[h, :L], V[h, :L], False, 0.5)
        np.testing.assert_array_equal(O[0, h], o[0])
        assert LSE[0, h] == lse[0]


def test_paged_shuffle_identical():
    q, kc, vc, table, lens, bs = _tiny_paged(4)
    perm = np.random.default_rng(9).permutation(kc.shape[0])
    kc2 = np.empty_like(kc)
    vc2 = np.empty_like(vc)
    kc2[perm] = kc
    vc2[perm] = vc
    t2 = np.where(table >= 0, perm[np.maximum(table, 0)], -1)
    O1, L1 = oracle.paged_decode(q, kc, vc, table, lens, bs, 0.5)
    O2, L2 = oracle.paged_decode(q, kc2, vc2, t2, lens, bs, 0.5)
    np.testing.assert_array_equal(O1, O2)
    np.testing.assert_array_equal(L1, L2)


def test_gather_rejects_bad_entry():
    q, kc, vc, table, lens, bs = _tiny_paged(5)
    table = table.copy()
    table[0, 1] = kc.shape[0]
    with pytest.raises(IndexError):
        oracle.paged_decode(q, kc, vc, table, lens, bs, 0.5, seqs=[0])


def test_merge_partials_any_split():
    """Split-KV merge: attention over disjoint key ranges, merged by LSE,
    equals attention over all keys, for every cut of a tiny sequence
    (checked against the one-shot definition)."""
    N, d = 9, 3
    q = _rand((1, d), 51)
    K, V = _rand((N, d), 52), _rand((N, d), 53)
    O_full, L_full = A.attention_head(q, K, V, False, 0.9)
    for cuts in itertools.chain.from_iterable(itertools.combinations(range(1, N), r) for r in range(0, 4)):
        bounds = [0, *cuts, N]
        Os, Ls = [], []
        for a, b in zip(bounds[:-1], bounds[1:]):
            o, l = A.attention_head(q, K[a:b], V[a:b], False, 0.9)
            Os.append(o)
            Ls.append(l)
        O, L = oracle.merge_partials(np.stack(Os), np.stack(Ls))
        np.testing.assert_allclose(O, O_full, atol=1e-13)
        np.testing.assert_allclose(L, L_full, atol=1e-13)
    # empty parts (-inf) contribute nothing; all-empty gives O = 0, LSE = -inf
    O, L = oracle.merge_partials(np.stack([O_full, np.zeros_like(O_full)]), np.stack([L_full, [-math.inf]]))
    np.testing.assert_allclose(O, O_full, atol=1e-15)
    O, L = oracle.merge_partials(np.zeros((2, 1, d)), np.full((2, 1), -math.inf))
    assert (O == 0).all() and L[0] == -math.inf


def test_attention_flops():
    """The algorithmic FLOP count is 4*d per visible (query, key) pair (2*d for
    q.k and 2*d for p*v).  The visible pairs are counted here two ways that do
    not use the formula: a double loop over (i, j) with the causal rule
    j <= i, and the nonzero entries of the oracle's materialised P on random
    inputs.  Then the two prefill workloads hit the rounded figures printed
    for them: 68.75 GFLOP (4 x 16 x 2048, d 128, causal) and 2.199 TFLOP
    (1 x 32 x 16384, d 128, causal)."""
    rng = np.random.default_rng(7)
    for N in range(1, 10):
        for causal in (False, True):
            loops = sum(1 for i in range(N) for j in range(N) if (j <= i or not causal))
            Q, K = rng.standard_normal((N, 4)), rng.standard_normal((N, 4))
            support = int(np.count_nonzero(oracle.softmax_probs(Q, K, causal, 0.5)))
            assert support == loops
            for B, H, d in ((1, 1, 4), (2, 3, 64)):
                assert oracle.attention_flops(B, H, N, d, causal) == 4 * d * B * H * loops
    assert round(oracle.attention_flops(4, 16, 2048, 128, True) / 1e9, 2) == 68.75
    assert round(oracle.attention_flops(1, 32, 16384, 128, True) / 1e12, 3) == 2.199
    assert round(oracle.attention_flops(1, 2, 128, 64, False) / 1e6, 2) == 8.39


# --------------------------------------------------------------------------
# planted mistakes: each must fail at least one pin
# --------------------------------------------------------------------------

def _mutant(kind):
    def attn(Q, K, V, causal, scale):
        Q, K, V = (np.asarray(x, dtype=np.float64) for x in (Q, K, V))
        B, H, Nq, _ = Q.shape
        Nk = K.shape[2]
        O = np.zeros((B, H, Nq, V.shape[3]))
        L = np.zeros((B, H, Nq))
        for b in range(B):
            for h in range(H):
                q, k, v = Q[b, h], K[b, h], V[b, h]
                s = (q @ k.T) * (1.0 if kind == "dropped_scale" else scale)
                if kind == "transposed":
                    s = (k @ q.T).T * scale if Nq != Nk else (k @ q.T) * scale
                if causal:
                    off = -1 if kind == "causal_off_by_one" else 0
                    s = np.where(np.arange(Nk)[None] <= np.arange(Nq)[:, None] + off, s, -np.inf)
                m = s.max(axis=1, keepdims=True)
                m = np.where(np.isfinite(m), m, 0)
                p = np.exp(s - m)
                l = p.sum(axis=1, keepdims=True)
                O[b, h] = (p @ v) / np.where(l > 0, l, 1)
                lse = np.log(np.where(l > 0, l, 1))[:, 0]
                L[b, h] = lse if kind == "lse_without_max" else lse + m[:, 0]
                if kind == "values_unnormalised":
                    O[b, h] = p @ v
        return O, L
    return attn


@pytest.mark.parametrize("kind", ["dropped_scale", "transposed", "causal_off_by_one",
                                  "lse_without_max", "values_unnormalised"])
def test_planted_mistakes_are_caught(kind):
    attn = _mutant(kind)
    caught = 0
    for pin in (pin_golden_dense, pin_torch_sdpa, pin_closed_forms):
        try:
            pin(attn)
        except AssertionError:
            caught += 1
    assert caught >= 1, f"planted mistake {kind!r} passed every pin"


def test_unmutated_copy_passes_pins():
    # the mutant scaffold itself is correct when no mistake is planted
    attn = _mutant("none")
    pin_golden_dense(attn)
    pin_torch_sdpa(attn)
    pin_closed_forms(attn)


# --------------------------------------------------------------------------
# KV-cache write and copy-on-write block copy
# --------------------------------------------------------------------------

def _pool(nb=10, H=2, bs=4, d=3, seed=60):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((nb, H, bs, d)), rng.standard_normal((nb, H, bs, d))


def test_kv_append_python_loops():
    """Token t goes to cache[table[s][pos // bs], h, pos % bs, :] for every
    head, element by element."""
    kc, vc = _pool()
    table = np.array([[3, 7, -1], [0, 9, 2]])
    rng = np.random.default_rng(61)
    seq_ids = np.array([0, 1, 1, 0, 1])
    pos = np.array([0, 5, 11, 6, 4])
    kn = rng.standard_normal((5, 2, 3))
    vn = rng.standard_normal((5, 2, 3))
    k2, v2, skipped = oracle.kv_append(kc, vc, table, kn, vn, seq_ids, pos, 4)
    assert skipped == []
    kref, vref = kc.copy(), vc.copy()
    for t in range(5):
        blk = table[seq_ids[t]][pos[t] // 4]
        for h in range(2):
            for c in range(3):
                kref[blk, h, pos[t] % 4, c] = kn[t, h, c]
                vref[blk, h, pos[t] % 4, c] = vn[t, h, c]
    np.testing.assert_array_equal(k2, kref)
    np.testing.assert_array_equal(v2, vref)
    assert (kc == _pool()[0]).all()  # input not modified


def test_kv_append_then_gather_round_trip():
    """Writing a sequence token by token then resolving the table by copy
    gives back exactly the written rows (gather_paged is pinned above)."""
    kc = np.zeros((8, 2, 4, 3))
    vc = np.zeros((8, 2, 4, 3))
    table = np.array([[5, 1, 6]])
    L = 10
    rng = np.random.default_rng(62)
    kn = rng.standard_normal((L, 2, 3))
    vn = rng.standard_normal((L, 2, 3))
    order = rng.permutation(L)  # order of writes does not matter
    k2, v2, _ = oracle.kv_append(kc, vc, table, kn[order], vn[order], np.zeros(L, int), order, 4)
    np.testing.assert_array_equal(oracle.gather_paged(k2, table[0], L, 4), kn.transpose(1, 0, 2))
    np.testing.assert_array_equal(oracle.gather_paged(v2, table[0], L, 4), vn.transpose(1, 0, 2))


def test_kv_append_skips_out_of_range():
    kc, vc = _pool()
    table = np.array([[3, 11]])  # 11 is outside the 10-block pool
    kn = np.ones((4, 2, 3))
    k2, v2, skipped = oracle.kv_append(kc, vc, table, kn, kn, np.array([0, 0, 1, 0]), np.array([1, 5, 0, 8]), 4)
    assert skipped == [1, 2, 3]  # bad table entry, bad sequence id, position past the table
    assert (k2[3, :, 1] == 1).all()
    k_check = kc.copy()
    k_check[3, :, 1] = 1
    np.testing.assert_array_equal(k2, k_check)


def test_block_copy_and_copy_on_write():
    kc, vc = _pool(seed=63)
    k2, v2, skipped = oracle.block_copy(kc, vc, [4, 2, 12], [6, 8, 0])
    assert skipped == [2]
    np.testing.assert_array_equal(k2[6], kc[4])
    np.testing.assert_array_equal(v2[8], vc[2])
    others = [b for b in range(10) if b not in (6, 8)]
    np.testing.assert_array_equal(k2[others], kc[others])
    # copy-on-write: two sequences share physical block 4; sequence 1 writes
    # into it, so the block is first copied to a free block 7 and its table
    # entry redirected; sequence 0 still sees the old contents
    table = np.array([[4, 1], [4, 3]])
    k3, v3, _ = oracle.block_copy(kc, vc, [4], [7])
    table[1, 0] = 7
    newk = np.full((1, 2, 3), 9.0)
    k4, v4, _ = oracle.kv_append(k3, v3, table, newk, newk, np.array([1]), np.array([2]), 4)
    g0 = oracle.gather_paged(k4, table[0], 4, 4)
    g1 = oracle.gather_paged(k4, table[1], 4, 4)
    np.testing.assert_array_equal(g0, kc[4])
    assert (g1[:, 2] == 9).all()
    np.testing.assert_array_equal(np.delete(g1, 2, axis=1), np.delete(kc[4], 2, axis=1))


def _refs_of(table, nb):
    refs = np.zeros(nb, dtype=np.int64)
    for b in np.asarray(table).ravel():
        if b >= 0:
            refs[b] += 1
    return refs


def test_cow_plan_hand_worked():
    """The copy-on-write step of the pages worked by hand: sequences 0 and 1
    share physical block 4 (count 2); sequence 1 writing its logical block 0
    takes free block 7, points its entry there and leaves block 4 to
    sequence 0 alone (count 1), which then writes in place: no second copy.
    A repeated write by sequence 1 finds its own block: no copy either."""
    table = np.array([[4, 1], [4, 3]])
    refs = np.array([0, 1, 0, 1, 2, 0, 0, 0, 0, 0])
    t, r, free, src, dst = oracle.cow_plan(table, refs, [9, 7], [(1, 0), (0, 0), (1, 0)])
    assert src == [4] and dst == [7] and free == [9]
    np.testing.assert_array_equal(t, [[4, 1], [7, 3]])
    np.testing.assert_array_equal(r, [0, 1, 0, 1, 1, 0, 0, 1, 0, 0])
    np.testing.assert_array_equal(table, [[4, 1], [4, 3]])  # inputs untouched
    # three sharers: the first two writers copy, the last one owns the block
    table = np.array([[5], [5], [5]])
    refs = _refs_of(table, 8)
    t, r, free, src, dst = oracle.cow_plan(table, refs, [1, 2, 3], [(0, 0), (2, 0), (1, 0)])
    assert src == [5, 5] and dst == [3, 2] and free == [1]
    np.testing.assert_array_equal(t, [[3], [5], [2]])
    np.testing.assert_array_equal(r, _refs_of(t, 8))


def test_cow_plan_invariants_and_contents():
    """Random shared-prefix tables: after the plan the counts are again the
    number of table references, every written entry is exclusive, unwritten
    entries keep their blocks, no free block is referenced, and copying the
    pairs (block_copy) leaves every sequence's logical contents as before."""
    rng = np.random.default_rng(90)
    for trial in range(30):
        S, mb, nb = 6, 5, 64
        pool = list(rng.permutation(nb))
        prefix = [pool.pop() for _ in range(2)]
        table = np.full((S, mb), -1)
        for s in range(S):
            n = int(rng.integers(1, mb + 1))
            for lb in range(n):
                table[s, lb] = prefix[lb] if lb < 2 and s % 3 else pool.pop()
        refs = _refs_of(table, nb)
        free = pool[:]
        live = [(s, lb) for s in range(S) for lb in range(mb) if table[s, lb] >= 0]
        writes = [live[i] for i in rng.integers(0, len(live), 12)]
        t, r, fr, src, dst = oracle.cow_plan(table, refs, free, writes)
        np.testing.assert_array_equal(r, _refs_of(t, nb))
        for s, lb in writes:
            assert r[t[s, lb]] == 1
        written = set(writes)
        for s, lb in live:
            if (s, lb) not in written:
                assert t[s, lb] == table[s, lb]
        assert not set(fr) & set(t[t >= 0].tolist())
        assert len(src) == len(set(dst)) == len(free) - len(fr)
        kc, vc = _pool(seed=100 + trial, nb=nb)
        k2, v2, skipped = oracle.block_copy(kc, vc, src, dst)
        assert skipped == []
        for s, lb in live:
            np.testing.assert_array_equal(k2[t[s, lb]], kc[table[s, lb]])
            np.testing.assert_array_equal(v2[t[s, lb]], vc[table[s, lb]])


def test_cow_plan_errors_and_planted_mistake():
    table = np.array([[4, -1], [4, 3]])
    refs = _refs_of(table, 8)
    for writes, free in [([(2, 0)], [7]), ([(0, 1)], [7]), ([(0, 0), (1, 0)], []), ([(0, 0)], [3]),
                         ([(0, 0)], [9])]:
        with pytest.raises(ValueError):
            oracle.cow_plan(table, refs, free, writes)
    bad = refs.copy()
    bad[3] = 0
    with pytest.raises(ValueError):
        oracle.cow_plan(table, bad, [7], [(1, 1)])

    def no_decrement(table, ref_counts, free_list, writes):  # a plausible slip: the source keeps its count
        t, r, f, src, dst = oracle.cow_plan(table, ref_counts, free_list, writes)
        for p in src:
            r[p] += 1
        return t, r, f, src, dst

    t, r, _, _, _ = no_decrement(np.array([[5], [5]]), np.array([0, 0, 0, 0, 0, 2]), [1], [(0, 0)])
    assert not (r == _refs_of(t, 6)).all()


def test_paged_decode_grouped_query_heads():
    """Grouped-query decode: query head h reads key/value head h // G.  Pinned
    against the multi-head oracle on a cache whose heads are repeated G times
    (each query head then has its own copy of its group's keys)."""
    q, kc, vc, table, lens, bs = _tiny_paged(21, S=5, H=2, d=3)
    G = 3
    qg = np.random.default_rng(22).standard_normal((5, 2 * G, 3))
    O, L = oracle.paged_decode(qg, kc, vc, table, lens, bs, 0.7)
    kr = np.repeat(kc, G, axis=1)
    vr = np.repeat(vc, G, axis=1)
    O2, L2 = oracle.paged_decode(qg, kr, vr, table, lens, bs, 0.7)
    np.testing.assert_array_equal(O, O2)
    np.testing.assert_array_equal(L, L2)
    with pytest.raises(ValueError):
        oracle.paged_decode(qg[:, :5], kc, vc, table, lens, bs, 0.7)


def test_paged_prefill_reduces_to_dense_causal_and_decode():
    """Paged prefill pins: (1) a sequence whose every token is new is dense
    causal attention on the gathered K/V (torch SDPA-pinned oracle); (2) one
    new token per sequence is paged decode; (3) n new tokens of a longer
    sequence equal the last n rows of dense causal attention over all L."""
    rng = np.random.default_rng(70)
    H, d, bs, nb = 2, 4, 4, 40
    kc = rng.standard_normal((nb, H, bs, d))
    vc = rng.standard_normal((nb, H, bs, d))
    table = rng.permutation(nb)[:30].reshape(3, 10)
    lens = np.array([13, 22, 9])
    n_new = np.array([13, 1, 4])
    cu = np.concatenate([[0], np.cumsum(n_new)])
    q = rng.standard_normal((cu[-1], H, d))
    O, L = oracle.paged_prefill(q, kc, vc, table, lens, cu, bs, 0.6)
    for s in range(3):
        Ks = oracle.gather_paged(kc, table[s], lens[s], bs)
        Vs = oracle.gather_paged(vc, table[s], lens[s], bs)
        for h in range(H):
            # queries placed at the last n positions of a length-L causal problem
            Qfull = np.zeros((lens[s], d))
            Qfull[lens[s] - n_new[s]:] = q[cu[s]:cu[s + 1], h]
            Od, Ld = A.attention_head(Qfull, Ks[h], Vs[h], True, 0.6)
            np.testing.assert_allclose(O[cu[s]:cu[s + 1], h], Od[lens[s] - n_new[s]:], atol=1e-13)
            np.testing.assert_allclose(L[cu[s]:cu[s + 1], h], Ld[lens[s] - n_new[s]:], atol=1e-13)
    Od, Ld = oracle.paged_decode(q[cu[1]:cu[2]], kc, vc, table[1:2], lens[1:2], bs, 0.6)
    np.testing.assert_allclose(O[cu[1]:cu[2]], Od, atol=1e-13)
    # (4) grouped heads: query heads 2h, 2h+1 read key/value head h, the same as
    # a multi-head cache holding each key/value head twice
    qg = rng.standard_normal((cu[-1], 2 * H, d))
    Og, Lg = oracle.paged_prefill(qg, kc, vc, table, lens, cu, bs, 0.6)
    Om, Lm = oracle.paged_prefill(qg, np.repeat(kc, 2, axis=1), np.repeat(vc, 2, axis=1), table, lens, cu, bs, 0.6)
    np.testing.assert_array_equal(Og, Om)
    np.testing.assert_array_equal(Lg, Lm)
    with pytest.raises(ValueError):
        oracle.paged_prefill(q, kc, vc, table, np.array([13, 22, 3]), cu, bs, 0.6)  # 4 new tokens, 3 cached
