"""The grouped decode's balanced schedule, restated on the host.

The kernel (decode_mma_kernel) lays the (sequence, key/value head) rows of
ceil(L / 16) tiles end to end, sequence-major, and gives worker w the tiles
[w c, (w + 1) c) with c = max(ceil(T / W), 8), W = 1184 workers.  A row cut
by worker boundaries leaves one partial per segment in slot worker + row;
the merge kernel reads a row's slots w0 + r .. w0 + r + nsplit - 1 with
w0 = row_begin // c and nsplit = (row_end - 1) // c - w0 + 1.  These checks
pin that arithmetic: every tile belongs to exactly one segment, a row's
segments come from consecutive workers, slots are unique and inside the
workspace the library sizes (1480 x 8 + rows x G partial rows), and the
merge's closed form names exactly the row's segments.
"""
import numpy as np
import pytest

WORKERS, MIN_TILES, MAX_WORKERS = 1184, 8, 1480


def _segments(lens, hkv):
    tiles = [-(-L // 16) if L > 0 else 0 for L in lens]
    starts = np.concatenate([[0], np.cumsum(tiles)]).astype(np.int64)
    T = int(starts[-1]) * hkv
    c = max(-(-T // WORKERS), MIN_TILES) if T else MIN_TILES
    nw = -(-T // c) if T else 0
    segs = []  # (worker, row, first tile, end tile) in line coordinates
    for w in range(nw):
        x, x_end = w * c, min(T, (w + 1) * c)
        while x < x_end:
            s = int(np.searchsorted(starts, x // hkv, side="right") - 1)
            nts = int(starts[s + 1] - starts[s])
            h = (x - hkv * int(starts[s])) // nts
            row_begin = hkv * int(starts[s]) + h * nts
            end = min(row_begin + nts, x_end)
            segs.append((w, s * hkv + h, x, end))
            x = end
    return tiles, starts, T, c, nw, segs


@pytest.mark.parametrize("seed,n,hkv,lo,hi", [(0, 64, 4, 128, 4096), (1, 64, 8, 0, 850), (2, 5, 1, 1, 20000),
                                              (3, 300, 2, 0, 40), (4, 7, 4, 0, 0), (5, 4100, 1, 0, 40),
                                              (6, 1, 1, 1, 16)])
def test_schedule_invariants(seed, n, hkv, lo, hi):
    lens = np.random.default_rng(seed).integers(lo, hi + 1, n).tolist()
    tiles, starts, T, c, nw, segs = _segments(lens, hkv)
    covered = np.zeros(T, dtype=np.int64)
    for _, _, a, b in segs:
        covered[a:b] += 1
    assert (covered == 1).all()
    assert nw <= WORKERS
    slots = set()
    by_row = {}
    for w, r, a, b in segs:
        by_row.setdefault(r, []).append(w)
        assert w + r not in slots
        slots.add(w + r)
    G = 8
    assert all(sl * G + G <= MAX_WORKERS * 8 + n * hkv * G for sl in slots)
    for r, ws in by_row.items():
        assert ws == list(range(ws[0], ws[0] + len(ws)))  # consecutive workers
        s, h = divmod(r, hkv)
        nts = tiles[s]
        row_begin = hkv * int(starts[s]) + h * nts
        w0 = row_begin // c
        nsplit = (row_begin + nts - 1) // c - w0 + 1
        assert ws[0] == w0 and len(ws) == nsplit
    # rows of empty sequences have no segment; all others have one at least
    assert set(by_row) == {s * hkv + h for s in range(n) if tiles[s] for h in range(hkv)}
