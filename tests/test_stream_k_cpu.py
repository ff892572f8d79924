"""Host-side checks of the stream-K work split of the attention kernels.

The split kernel lays the tiles of all units (sequence b, kv head, group of
8 query heads) end to end: sequence b's units start at prefix[b], each unit
of sequence b holds T_b = ceil(seq_b / 16) tiles, and the W tiles are cut into
G equal contiguous ranges, CTA c taking [floor(c W / G), floor((c+1) W / G)).
A CTA walks its range unit by unit and writes one partial per piece
(segment) to slot c + u. The reduce finds the CTAs covering unit u
arithmetically (tile x lies in CTA floor(((x+1) G - 1) / W)) and steps their
range starts as quotient and remainder of c W / G.

These tests restate that arithmetic in Python and check the properties the
kernels rely on, over random ragged batches (lengths from 0 to several
tiles, grids larger and smaller than the tile count):
  * every tile lies in exactly one CTA, and the closed form finds it;
  * a unit's covering CTAs cf..cl are exactly the CTAs whose non-empty
    ranges meet the unit;
  * no two segments share a partial slot, and slots stay below G + units;
  * the quotient/remainder walk equals direct division.
"""
import numpy as np
import pytest


def prefix_of(seq_tiles, upb):
    pre = [0]
    for t in seq_tiles:
        pre.append(pre[-1] + t * upb)
    return pre


def segments(W, G, pre, seq_tiles, upb):
    """(cta, unit, first tile, end tile) of every segment, as the split kernel walks."""
    out = []
    for c in range(G):
        x0, x1 = c * W // G, (c + 1) * W // G
        x = x0
        while x < x1:
            b = max(i for i in range(len(seq_tiles)) if pre[i] <= x and seq_tiles[i] > 0)
            T = seq_tiles[b]
            j = (x - pre[b]) // T
            U0 = pre[b] + j * T
            se = min(T, x1 - U0)
            out.append((c, b * upb + j, x, U0 + se))
            x = U0 + se
    return out


def covering(W, G, U0, T):
    cf = ((U0 + 1) * G - 1) // W
    cl = ((U0 + T) * G - 1) // W
    return cf, cl


def walk(W, G, cf, cl):
    """Range starts of CTAs cf..cl+1 stepped as quotient and remainder."""
    wq, wr = W // G, W - (W // G) * G
    q = cf * W // G
    r = cf * W - q * G
    starts = [q]
    for _ in range(cf, cl + 1):
        qn, rn = q + wq, r + wr
        if rn >= G:
            qn, rn = qn + 1, rn - G
        starts.append(qn)
        q, r = qn, rn
    return starts


def random_case(rng):
    B = int(rng.integers(1, 9))
    upb = int(rng.integers(1, 5))
    seq_tiles = [int(t) for t in rng.integers(0, 7, size=B)]
    if sum(seq_tiles) == 0:
        seq_tiles[int(rng.integers(0, B))] = 1
    pre = prefix_of(seq_tiles, upb)
    W = pre[-1]
    G = int(rng.integers(1, 3 * W + 2))
    return B, upb, seq_tiles, pre, W, G


@pytest.mark.parametrize("seed", range(8))
def test_stream_k_partition_properties(seed):
    rng = np.random.default_rng(seed)
    for _ in range(250):
        B, upb, seq_tiles, pre, W, G = random_case(rng)
        # every tile in exactly one CTA, found by the closed form
        owner = np.full(W, -1)
        for c in range(G):
            lo, hi = c * W // G, (c + 1) * W // G
            assert np.all(owner[lo:hi] == -1)
            owner[lo:hi] = c
        assert np.all(owner >= 0)
        x = np.arange(W)
        assert np.array_equal(((x + 1) * G - 1) // W, owner)
        # segments: one unit each, slots unique and bounded
        segs = segments(W, G, pre, seq_tiles, upb)
        slots = [c + u for c, u, _, _ in segs]
        assert len(slots) == len(set(slots))
        assert max(slots) < G + B * upb
        covered = np.zeros(W, int)
        for c, u, a, e in segs:
            assert owner[a] == c and owner[e - 1] == c and a < e
            covered[a:e] += 1
        assert np.all(covered == 1)
        # covering CTAs of each unit, and the reduce's walk over them
        for b in range(B):
            T = seq_tiles[b]
            if T == 0:
                continue
            for j in range(upb):
                u = b * upb + j
                U0 = pre[b] + j * T
                cf, cl = covering(W, G, U0, T)
                starts = walk(W, G, cf, cl)
                assert starts == [c * W // G for c in range(cf, cl + 2)]
                live = [c for c in range(cf, cl + 1) if starts[c - cf + 1] != starts[c - cf]]
                writers = sorted(c for c, uu, _, _ in segs if uu == u)
                assert live == writers


def test_walk_matches_division_on_large_grids():
    rng = np.random.default_rng(123)
    for _ in range(2000):
        G = int(rng.integers(1, 1200))
        W = int(rng.integers(1, 10 ** 8))
        cf = int(rng.integers(0, G))
        cl = int(rng.integers(cf, min(G, cf + 300)))
        assert walk(W, G, cf, cl) == [c * W // G for c in range(cf, cl + 2)]
