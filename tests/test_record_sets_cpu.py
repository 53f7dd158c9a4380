"""Split records of the tensor-core decode: the sets the combine reads are exactly the sets the
decode CTAs write (no GPU).

The decode kernels walk a flattened (sequence, 128-token tile) space: the G CTAs form G / parts
groups, group g takes tiles [floor(total g / groups), floor(total (g + 1) / groups)), and a CTA
writes one record set per sequence its range touches, with id (g + b) parts + part.  The combine
finds sequence b's groups from the owner of its first and last tiles,
owner(x) = floor(((x + 1) groups - 1) / total), and skips groups whose range is empty.  The
workspace is not cleared between calls, so any record set read but not written would bring stale
bytes into the output; this checks the two index schemes against each other over seeded batches
with empty sequences, fewer tiles than groups and 1, 4 or 8 head parts.
"""

import numpy as np
import pytest

TILE = 128


def _prefix(lens):
    tiles = [(n + TILE - 1) // TILE for n in lens]
    return np.concatenate([[0], np.cumsum(tiles)]).astype(np.int64), tiles


def _written(P, G, parts):
    """{(b, part): sorted group ids} written by the walk: each group walks its tile range."""
    B, total, groups = len(P) - 1, int(P[-1]), G // parts
    out = {}
    for g in range(groups):
        x, x1 = total * g // groups, total * (g + 1) // groups
        for t in range(x, x1):
            b = int(np.searchsorted(P, t, side="right") - 1)  # largest b with P[b] <= t
            assert P[b] <= t < P[b + 1]
            for part in range(parts):
                s = out.setdefault((b, part), [])
                if not s or s[-1] != g:
                    s.append(g)
    return out


def _read(P, tiles, b, G, parts):
    """Groups the combine reads for sequence b (any part): g0 .. g1 minus empty ranges."""
    total, groups = int(P[-1]), G // parts
    if tiles[b] == 0 or total == 0:
        return []
    x0, x1 = int(P[b]), int(P[b]) + tiles[b] - 1
    g0 = ((x0 + 1) * groups - 1) // total
    g1 = ((x1 + 1) * groups - 1) // total
    return [g for g in range(g0, g1 + 1) if total >= groups or total * (g + 1) // groups > total * g // groups]


def _owner_ok(total, groups):
    for x in range(total):
        g = ((x + 1) * groups - 1) // total
        assert total * g // groups <= x < total * (g + 1) // groups, (x, total, groups)


@pytest.mark.parametrize("G,parts", [(148, 1), (148, 4), (144, 8), (7, 1), (8, 4)])
def test_records_read_are_exactly_the_records_written(G, parts):
    rng = np.random.default_rng(0x11A + G * 31 + parts)
    for _ in range(300):
        B = int(rng.integers(1, 40))
        kind = rng.integers(0, 3)
        if kind == 0:  # mostly short, many empty: fewer tiles than groups
            lens = rng.integers(0, 3 * TILE, size=B)
        elif kind == 1:  # long and ragged
            lens = rng.integers(0, 40 * TILE, size=B)
        else:  # tile boundaries and zeros
            lens = rng.choice([0, 1, TILE - 1, TILE, TILE + 1, 5 * TILE], size=B)
        P, tiles = _prefix(lens)
        total, groups = int(P[-1]), G // parts
        if total:
            _owner_ok(total, groups)
        w = _written(P, G, parts)
        for b in range(B):
            r = _read(P, tiles, b, G, parts)
            for part in range(parts):
                assert r == w.get((b, part), []), (b, part, list(lens), G, parts)
        # record ids of different (group, sequence) pairs never collide
        ids = [(g + b) * parts + p for (b, p), gs in w.items() for g in gs]
        assert len(ids) == len(set(ids))
        assert all(0 <= i < G + parts * B for i in ids)  # inside the workspace's record area
