"""The prefill kernel's work units, restated on the host.

prefill_bf16_kernel gives each persistent CTA c of G the units
u = r G + (c, or G - 1 - c on odd rounds r) for r = 0, 1, ... while
u < n_units (snake order).  A dense unit is (128-row query block pair blk,
head bh): blk = nblk - 1 - u // BH when causal (longest first), u // BH
otherwise, bh = u % BH; its two query tiles are rows qrow0 = 256 blk ..
+ 127 and + 128 .. + 255, and in a bf16 causal unit tile 0 takes the later
128 rows (the one with the extra diagonal key tile).  A paged unit is
(sequence s, query block qb, query head h) with u = s (nqb Hq) + ... and the
later query blocks of a sequence first.  Tile i needs the key tiles
0 .. n_i - 1: n_i = min((pos0 + row0_i + 127) // 128 + 1, ceil(L / 128))
when causal, ceil(L / 128) otherwise, and 0 for a tile with no rows.

These checks pin that arithmetic: every unit goes to exactly one CTA, every
(head, query row) to exactly one tile, n_i is exactly the number of key
tiles the tile's last row attends (so no needed key tile is skipped and no
tile past the diagonal is computed), tile 0 of a later-first causal unit
never has fewer key tiles than tile 1 when both have rows (in the last,
partial query block tile 0 can be empty), and the snake order keeps the most
loaded CTA within a few percent of the mean at the 2k workload.
"""
import numpy as np
import pytest

BM = BN = 128
NQ = 2


def _snake_unit(r, c, G, n_units):
    u = r * G + ((G - 1 - c) if (r & 1) else c)
    return u if u < n_units else -1


def _tile_counts(pos0, qrow0, nq, L, causal, later_first):
    n_kv_all = -(-L // BN)
    row0 = [qrow0 + (BM if later_first else 0), qrow0 + (0 if later_first else BM)]
    n = []
    for r0 in row0:
        if r0 >= nq:
            n.append(0)
        else:
            n.append(min((pos0 + r0 + BM - 1) // BN + 1, n_kv_all) if causal else n_kv_all)
    return row0, n


def _dense_unit(u, BH, N, causal, later_first):
    nblk = -(-N // (NQ * BM))
    blk = (nblk - 1 - u // BH) if causal else (u // BH)
    bh = u % BH
    qrow0 = NQ * BM * blk
    row0, n = _tile_counts(0, qrow0, N, N, causal, later_first)
    return bh, row0, n


def _walk(n_units, G):
    owner = {}
    for c in range(G):
        r = 0
        while True:
            u = _snake_unit(r, c, G, n_units)
            if u < 0:
                break
            assert u not in owner
            owner[u] = c
            r += 1
    return owner


@pytest.mark.parametrize("BH,N,causal,later_first", [(64, 2048, True, True), (64, 2048, True, False),
                                                     (64, 2048, False, False), (32, 16384, True, True),
                                                     (3, 1000, True, True), (5, 300, False, False),
                                                     (1, 1, True, True), (7, 257, True, True)])
def test_dense_units_cover_rows_once_with_exact_key_tiles(BH, N, causal, later_first):
    nblk = -(-N // (NQ * BM))
    n_units = nblk * BH
    G = min(n_units, 148)
    owner = _walk(n_units, G)
    assert sorted(owner) == list(range(n_units))
    covered = np.zeros((BH, N), dtype=np.int64)
    for u in range(n_units):
        bh, row0, n = _dense_unit(u, BH, N, causal, later_first)
        for i in range(NQ):
            rows = range(row0[i], min(row0[i] + BM, N))
            if n[i] == 0:
                assert len(rows) == 0
                continue
            covered[bh, rows.start:rows.stop] += 1
            # the key tiles the tile's rows attend: 0 .. max over rows of (last key // BN)
            need = max(((q if causal else N - 1) // BN) for q in rows) + 1
            assert n[i] == need
        if causal and later_first and n[0] > 0 and n[1] > 0:
            assert n[0] >= n[1]
        if causal and later_first and n[0] == 0:
            # the last, partial query block: the later 128 rows lie past N
            assert row0[0] >= N and (n[1] > 0) == (row0[1] < N)
    assert (covered == 1).all()


def test_dense_2k_snake_balance():
    """At the 2k causal workload the snake order leaves the most loaded CTA
    (in key steps of the longer tile, which set a unit's length) within 5 %
    of the mean."""
    BH, N = 64, 2048
    nblk = N // (NQ * BM)
    n_units = nblk * BH
    G = 148
    load = np.zeros(G)
    for u, c in _walk(n_units, G).items():
        _, _, n = _dense_unit(u, BH, N, True, True)
        load[c] += max(n)
    assert load.max() / load.mean() <= 1.05


@pytest.mark.parametrize("seed", range(6))
def test_paged_units_cover_new_tokens_once(seed):
    """Paged (chunked) prefill: sequences with n_s new tokens after L_s - n_s
    cached ones; the units cover every (sequence, query head, new token)
    exactly once, and each tile's key tiles reach exactly the last key its
    rows attend (position L_s - n_s + row)."""
    rng = np.random.default_rng(seed)
    S, Hq = int(rng.integers(1, 5)), int(rng.integers(1, 4))
    nq = rng.integers(0, 700, S)
    L = nq + rng.integers(0, 900, S)
    nqb = max(1, -(-int(nq.max()) // (NQ * BM)))
    per_seq = nqb * Hq
    n_units = S * per_seq
    G = min(n_units, 148)
    assert sorted(_walk(n_units, G)) == list(range(n_units))
    covered = [np.zeros((Hq, int(n)), dtype=np.int64) for n in nq]
    for u in range(n_units):
        s = u // per_seq
        rem = u - s * per_seq
        qb = nqb - 1 - rem // Hq
        h = rem % Hq
        pos0 = int(L[s] - nq[s])
        row0, n = _tile_counts(pos0, NQ * BM * qb, int(nq[s]), int(L[s]), True, True)
        for i in range(NQ):
            rows = range(row0[i], min(row0[i] + BM, int(nq[s])))
            if n[i] == 0:
                assert len(rows) == 0
                continue
            covered[s][h, rows.start:rows.stop] += 1
            assert n[i] == (pos0 + rows.stop - 1) // BN + 1
    for c in covered:
        assert (c == 1).all()
