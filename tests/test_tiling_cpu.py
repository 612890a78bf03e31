"""The triangular MaxSim tile order, checked exhaustively on the host.

The CTA-pair MaxSim kernel (avey_maxsim2.cu) computes only the 256 x 256
tiles on or right of the diagonal of 256-row blocks.  Per tile, CTA r of the
pair holds rows r*128 .. r*128+127, and each of its two 128-column halves
writes row-direction scores for its candidate splits and, right of the
diagonal, the mirrored column-direction scores.  This transcribes the
kernel's slot decode and write rules (decode_pair, pair_write) and checks
that every ordered split pair (t, c) is written exactly once, for many
sequence lengths and split sizes, and that every index stays in range.  The
kernel's roles walk their slots incrementally (PairCursor); a mirror of that
walk is checked against the closed-form decode.
"""
import itertools
import math

import pytest


GP = 32  # 256-row blocks per group (kGroup)


def _prefix_pair(g, tn):
    return GP * g * tn - GP * GP * g * (g - 1) // 2


def _decode_pair(x, tn):
    A = GP * tn + GP * GP / 2.0
    disc = A * A - 2.0 * GP * GP * x
    g = max(int((A - math.sqrt(max(disc, 0.0))) / (GP * GP)), 0)
    while g > 0 and _prefix_pair(g, tn) > x:
        g -= 1
    while _prefix_pair(g + 1, tn) <= x and (g + 1) * GP < tn:
        g += 1
    rem = x - _prefix_pair(g, tn)
    rows_g = min(GP, tn - g * GP)
    nt = g * GP + rem // rows_g
    mt = g * GP + rem % rows_g
    return mt, nt, nt >= mt


def _coverage_pair(N, S):
    n = -(-N // S)
    R = n * S
    tn = -(-R // 256)
    slots = sum(min(GP, tn - g * GP) * (tn - g * GP) for g in range(-(-tn // GP)))
    TS = CB = 128 // S
    seen, tiles = {}, set()
    for x in range(slots):
        mt, nt, ok = _decode_pair(x, tn)
        assert 0 <= mt < tn and 0 <= nt < tn
        if not ok:
            continue
        assert (mt, nt) not in tiles
        tiles.add((mt, nt))
        for rank, half in itertools.product(range(2), range(2)):
            t0, c0 = (mt * 256 + rank * 128) // S, (nt * 256 + half * 128) // S
            for ts, cl in itertools.product(range(TS), range(CB)):
                t, c = t0 + ts, c0 + cl
                if t < n and c < n:
                    seen[(t, c)] = seen.get((t, c), 0) + 1
                    if nt > mt:
                        seen[(c, t)] = seen.get((c, t), 0) + 1
    bad = [(t, c) for t in range(n) for c in range(n) if seen.get((t, c), 0) != 1]
    return bad, len(tiles), tn * tn


@pytest.mark.parametrize("N", [64, 100, 255, 256, 257, 1000, 2053, 4096, 5000, 16384, 33000])
@pytest.mark.parametrize("S", [32, 64, 128])
def test_pair_every_ordered_pair_written_once(N, S):
    bad, _, _ = _coverage_pair(N, S)
    assert not bad, bad[:5]


def test_pair_long_workload_tiles():
    bad, tiles, full = _coverage_pair(98304, 64)
    assert not bad
    assert full == 384 * 384 and tiles == 384 * 385 // 2


@pytest.mark.parametrize("nparts", [2, 3, 8])
@pytest.mark.parametrize("N,S", [(4096, 64), (5000, 32), (2500, 128)])
def test_pair_parts_partition_the_entries(N, S, nparts):
    # avey_maxsim_part: part p takes the tiles t with t % nparts == p of the
    # same slot order; every ordered split pair is written by exactly one part
    n = -(-N // S)
    tn = -(-(n * S) // 256)
    slots = sum(min(GP, tn - g * GP) * (tn - g * GP) for g in range(-(-tn // GP)))
    TS = CB = 128 // S
    owner = {}
    for x in range(slots):
        mt, nt, ok = _decode_pair(x, tn)
        if not ok:
            continue
        part = x % nparts
        for rank, half in itertools.product(range(2), range(2)):
            t0, c0 = (mt * 256 + rank * 128) // S, (nt * 256 + half * 128) // S
            for ts, cl in itertools.product(range(TS), range(CB)):
                t, c = t0 + ts, c0 + cl
                if t < n and c < n:
                    for key in ((t, c), (c, t)) if nt > mt else ((t, c),):
                        assert key not in owner
                        owner[key] = part
    assert len(owner) == n * n


class _Cursor:
    """The kernel's incremental walk (PairCursor): the first slot is located
    with the closed-form decode, then each step moves the in-group offset on
    and crosses whole groups and sequences."""

    def __init__(self, first, tn, slots, num_tiles):
        self.tn, self.num_tiles = tn, num_tiles
        self.tile = first
        self.b = first // slots
        x = first - self.b * slots
        A = GP * tn + GP * GP / 2.0
        disc = A * A - 2.0 * GP * GP * x
        g = max(int((A - math.sqrt(max(disc, 0.0))) / (GP * GP)), 0)
        while g > 0 and _prefix_pair(g, tn) > x:
            g -= 1
        while _prefix_pair(g + 1, tn) <= x and (g + 1) * GP < tn:
            g += 1
        self.g, self.x = g, x - _prefix_pair(g, tn)
        self._size()

    def _size(self):
        self.rows = min(GP, self.tn - self.g * GP)
        self.size = self.rows * (self.tn - self.g * GP)

    def next(self, step):
        self.tile += step
        if self.tile >= self.num_tiles:
            return
        self.x += step
        while self.x >= self.size:
            self.x -= self.size
            self.g += 1
            if self.g * GP >= self.tn:
                self.g, self.b = 0, self.b + 1
            self._size()

    def tile_of(self):
        q = self.x // self.rows
        return self.g * GP + (self.x - q * self.rows), self.g * GP + q


@pytest.mark.parametrize("tn", [1, 2, 31, 32, 33, 64, 100, 384, 513])
@pytest.mark.parametrize("B", [1, 3])
@pytest.mark.parametrize("step", [1, 7, 74, 148, 592])
def test_cursor_walks_the_decoded_order(tn, B, step):
    # every pair's incremental walk visits exactly the slots the closed-form
    # decode gives, sequence by sequence, and the pairs together visit each
    # slot once
    slots = sum(min(GP, tn - g * GP) * (tn - g * GP) for g in range(-(-tn // GP)))
    num = B * slots
    seen = 0
    for first in range(min(step, num)):
        c = _Cursor(first, tn, slots, num)
        while c.tile < num:
            x = c.tile % slots
            mt, nt, _ = _decode_pair(x, tn)
            assert (c.b, c.tile_of()) == (c.tile // slots, (mt, nt)), (first, c.tile)
            seen += 1
            c.next(step)
    assert seen == num
