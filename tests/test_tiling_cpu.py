"""The triangular MaxSim tile order, checked exhaustively on the host.

The tcgen05 MaxSim kernel computes only the 128x256 tiles that reach the
diagonal of 128-row blocks and writes, per tile, row-direction scores for the
column blocks on or right of the diagonal and column-direction (mirrored)
scores for the blocks right of it.  This transcribes the kernel's slot decode
and write rules (avey_tc.cu: decode_tile, epi_maxsim_sym_write) and checks
that every ordered split pair (t, c) is written exactly once, for many
sequence lengths and split sizes, and that every index stays in range.
"""
import itertools
import math

import pytest

G = 64  # row tiles per group (kSymGroup)


def _prefix(g, tn):
    return G * g * tn - (G // 2) * G * g * (g - 1) // 2


def _decode(x, tm, tn):
    A = G * tn + (G // 2) * G / 2.0
    disc = A * A - 2.0 * (G // 2) * G * x
    g = max(int((A - math.sqrt(max(disc, 0.0))) / ((G // 2) * G)), 0)
    while g > 0 and _prefix(g, tn) > x:
        g -= 1
    while _prefix(g + 1, tn) <= x and (g + 1) * G < tm:
        g += 1
    rem = x - _prefix(g, tn)
    rows_g = min(G, tm - g * G)
    nt = g * (G // 2) + rem // rows_g
    mt = g * G + rem % rows_g
    return mt, nt, 2 * nt + 1 >= mt


def _coverage(N, S):
    n = -(-N // S)
    R = n * S
    tm, tn = -(-R // 128), -(-R // 256)
    slots = sum(min(G, tm - g * G) * (tn - g * (G // 2)) for g in range(-(-tm // G)))
    TS, NC, CB = 128 // S, 256 // S, 128 // S
    seen, tiles = {}, set()
    for x in range(slots):
        mt, nt, ok = _decode(x, tm, tn)
        assert 0 <= mt < tm and 0 <= nt < tn
        if not ok:
            continue
        assert (mt, nt) not in tiles
        tiles.add((mt, nt))
        for ts, cs in itertools.product(range(TS), range(NC)):
            if 2 * nt + (cs * S) // 128 < mt:
                continue
            t, c = mt * TS + ts, nt * NC + cs
            if t < n and c < n:
                seen[(t, c)] = seen.get((t, c), 0) + 1
        for kb in range(2):
            K = 2 * nt + kb
            if K <= mt:
                continue
            for ts, cl in itertools.product(range(TS), range(CB)):
                t, c = mt * TS + ts, K * CB + cl
                if t < n and c < n:
                    seen[(c, t)] = seen.get((c, t), 0) + 1
    bad = [(t, c) for t in range(n) for c in range(n) if seen.get((t, c), 0) != 1]
    return bad, len(tiles), tm * tn


@pytest.mark.parametrize("N", [64, 100, 255, 256, 1000, 2053, 4096, 5000, 16384, 33000])
@pytest.mark.parametrize("S", [32, 64, 128])
def test_every_ordered_pair_written_once(N, S):
    bad, _, _ = _coverage(N, S)
    assert not bad, bad[:5]


def test_long_workload_computes_half_the_tiles():
    bad, tiles, full = _coverage(98304, 64)
    assert not bad
    assert tiles == 147840 and full == 294912
