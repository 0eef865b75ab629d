"""The grouped decode's balanced schedule, restated on the host.

The kernel (decode_mma_kernel) lays the (sequence, key/value head) rows of
ceil(L / 16) tiles end to end, sequence-major, T tiles in all, and gives
worker w of nw = min(W, max(1, T // 8)) the tiles
[w T // nw, (w + 1) T // nw), W being the launch's math warps (8 per CTA,
one CTA per SM, at most 1480).  A row cut by worker boundaries leaves one
partial per segment in slot worker + row; the merge kernel reads a row's
slots w0 + r .. w0 + r + nsplit - 1 with w0 = worker_of(row_begin),
nsplit = worker_of(row_end - 1) - w0 + 1 and worker_of(x) =
((x + 1) nw - 1) // T.  These checks pin that arithmetic: every tile
belongs to exactly one segment, every worker has a run (none idles while
another works) no shorter than 8 tiles unless T is, runs differ by at most
one tile, a row's segments come from consecutive workers, slots are unique
and inside the workspace the library sizes (1480 x 8 + rows x G partial
rows), worker_of inverts the run starts, and the merge's closed form names
exactly the row's segments.
"""
import numpy as np
import pytest

MIN_TILES, MAX_WORKERS = 8, 1480


def _nw(T, W):
    return max(1, min(W, T // MIN_TILES))


def _run_begin(w, T, nw):
    return w * T // nw


def _worker_of(x, T, nw):
    return ((x + 1) * nw - 1) // T


def _segments(lens, hkv, W):
    tiles = [-(-L // 16) if L > 0 else 0 for L in lens]
    starts = np.concatenate([[0], np.cumsum(tiles)]).astype(np.int64)
    T = int(starts[-1]) * hkv
    nw = _nw(T, W) if T else 0
    segs = []  # (worker, row, first tile, end tile) in line coordinates
    for w in range(nw):
        x, x_end = _run_begin(w, T, nw), _run_begin(w + 1, T, nw)
        while x < x_end:
            s = int(np.searchsorted(starts, x // hkv, side="right") - 1)
            nts = int(starts[s + 1] - starts[s])
            h = (x - hkv * int(starts[s])) // nts
            row_begin = hkv * int(starts[s]) + h * nts
            end = min(row_begin + nts, x_end)
            segs.append((w, s * hkv + h, x, end))
            x = end
    return tiles, starts, T, nw, segs


@pytest.mark.parametrize("seed,n,hkv,lo,hi,W", [(0, 64, 4, 128, 4096, 1184), (1, 64, 8, 0, 850, 1184),
                                                (2, 5, 1, 1, 20000, 1184), (3, 300, 2, 0, 40, 1184),
                                                (4, 7, 4, 0, 0, 1184), (5, 4100, 1, 0, 40, 1184),
                                                (6, 1, 1, 1, 16, 1184), (7, 64, 4, 128, 4096, 1040),
                                                (8, 200, 8, 1, 9000, 1480)])
def test_schedule_invariants(seed, n, hkv, lo, hi, W):
    lens = np.random.default_rng(seed).integers(lo, hi + 1, n).tolist()
    tiles, starts, T, nw, segs = _segments(lens, hkv, W)
    covered = np.zeros(T, dtype=np.int64)
    for _, _, a, b in segs:
        covered[a:b] += 1
    assert (covered == 1).all()
    assert nw <= W
    if T:
        runs = [_run_begin(w + 1, T, nw) - _run_begin(w, T, nw) for w in range(nw)]
        assert max(runs) - min(runs) <= 1
        assert min(runs) >= min(T, MIN_TILES)
        # no worker idles while another has more than its 8-tile floor twice over
        assert nw == W or min(runs) < 2 * MIN_TILES
        # worker_of inverts the run starts
        for w in range(nw):
            b0, b1 = _run_begin(w, T, nw), _run_begin(w + 1, T, nw)
            assert _worker_of(b0, T, nw) == w and _worker_of(b1 - 1, T, nw) == w
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
        w0 = _worker_of(row_begin, T, nw)
        nsplit = _worker_of(row_begin + nts - 1, T, nw) - w0 + 1
        assert ws[0] == w0 and len(ws) == nsplit
    # rows of empty sequences have no segment; all others have one at least
    assert set(by_row) == {s * hkv + h for s in range(n) if tiles[s] for h in range(hkv)}


def test_worker_of_brute_force():
    """worker_of(x) = ((x + 1) nw - 1) // T is the run holding x, for every
    tile of small schedules (and runs of one tile)."""
    for T in range(1, 200):
        for nw in range(1, min(T, 40) + 1):
            owner = np.empty(T, dtype=np.int64)
            for w in range(nw):
                owner[_run_begin(w, T, nw):_run_begin(w + 1, T, nw)] = w
            assert all(_worker_of(x, T, nw) == owner[x] for x in range(T))
