"""The kernels' tile schedules, restated on the host and checked against
brute-force visibility (CPU only; the GPU parity tests check the kernels).

Every kernel decides which 128 x 128 (query, key) tiles to compute from the
per-token visibility bounds: query i sees keys lo(i)..hi(i), key j is seen by
queries imin(j)..imax(j), all four non-decreasing in the position. The tiles to
visit in one run of consecutive positions are then an interval. This file
writes those rules out in Python, the way the kernels apply them, and checks on
small layouts (contiguous and zigzag, several P, causal or not, sliding
windows, packed documents) that:
* the bounds table matches the definition of visibility, and is monotone;
* no tile with a visible pair is ever skipped, no tile is visited twice, and
  each visited tile's class (masked or full) is the true one;
* the backward schedules visit exactly the tiles with a visible pair;
* the all-gather and one-step forward schedules cover the same pairs as the
  ring, the one-step schedule only within the owner's block.
"""
import random

import numpy as np
import pytest

T = 128
SKIP, MASK, FULL = 0, 1, 2


def ceil_div128(x):
    return -((-x) >> 7)


def bounds_table(S, causal, window, cu):
    """Per token (lo, hi, imin, imax) as the kernels' bounds (documents
    [cu[d], cu[d+1]); a window counts keys, itself included)."""
    cu = [0, S] if cu is None else cu
    out = []
    d = 0
    for i in range(S):
        while cu[d + 1] <= i:
            d += 1
        ds, de = cu[d], cu[d + 1]
        lo, imax = ds, de - 1
        if causal and window:
            lo, imax = max(lo, i - window + 1), min(imax, i + window - 1)
        out.append((lo, i if causal else de - 1, i if causal else ds, imax))
    return out


def visible(S, causal, window, cu, i, j):
    cu = [0, S] if cu is None else cu
    doc = lambda x: max(n for n in range(len(cu) - 1) if cu[n] <= x)
    if doc(i) != doc(j):
        return False
    if causal and j > i:
        return False
    return not (causal and window and j <= i - window)


def class_from_bounds(first, last, p):
    """Class of the tile at positions p..p+127 for the row (or column) range
    whose first and last bounds are given."""
    if p > last[1] or p + T - 1 < first[0]:
        return SKIP
    return FULL if (p >= last[0] and p + T - 1 <= first[1]) else MASK


class Layout:
    """Rank-major slot <-> natural position (rank i: chunks i and 2P-1-i)."""

    def __init__(self, S, P, zigzag):
        self.S, self.P, self.L, self.zigzag = S, P, S // P, zigzag
        self.c = S // (2 * P) if zigzag else S // P

    def pos_of_slot(self, x):
        if not self.zigzag:
            return x
        i, u = divmod(x, self.L)
        return i * self.c + u if u < self.c else (2 * self.P - 1 - i) * self.c + (u - self.c)

    def slot_of_pos(self, x):
        if not self.zigzag:
            return x
        k, off = divmod(x, self.c)
        return k * self.L + off if k < self.P else (2 * self.P - 1 - k) * self.L + self.c + off

    def runs(self, r):
        """(tiles, first slot, first position) of each run of owner r's block."""
        tiles = (self.c if self.zigzag else self.L) // T
        for run in range(2 if self.zigzag else 1):
            p0 = ((r * self.c if run == 0 else (2 * self.P - 1 - r) * self.c) if self.zigzag
                  else r * self.L)
            yield tiles, r * self.L + run * self.c, p0


def interval(lo, hi, p0, tiles):
    return range(max(0, ceil_div128(lo - (T - 1) - p0)), min(tiles, max(((hi - p0) >> 7) + 1, 0)))


def fwd_ring(lay, tab, rank, pos0, pos1):
    lo, hi = min(tab[pos0][0], tab[pos1][0]), max(tab[pos0 + T - 1][1], tab[pos1 + T - 1][1])
    out = []
    for t in range(lay.P):
        for tiles, s0, p0 in lay.runs((rank - t) % lay.P):
            out += [(s0 + u * T, p0 + u * T) for u in interval(lo, hi, p0, tiles)]
    return out


def fwd_gathered(lay, tab, pos0, pos1):
    lo, hi = min(tab[pos0][0], tab[pos1][0]), max(tab[pos0 + T - 1][1], tab[pos1 + T - 1][1])
    return [(u * T, u * T) for u in interval(lo, hi, 0, lay.S // T)]


def fwd_step(lay, tab, owner, pos0, pos1):
    """(row within the owner's block, position) of the tiles one step visits."""
    lo, hi = min(tab[pos0][0], tab[pos1][0]), max(tab[pos0 + T - 1][1], tab[pos1 + T - 1][1])
    out = []
    for tiles, s0, p0 in lay.runs(owner):
        s0 -= owner * lay.L
        out += [(s0 + u * T, p0 + u * T) for u in interval(lo, hi, p0, tiles)]
    return out


def bwd_keys(lay, tab, rank, qpos):
    """dQ: key tiles of one query tile, ring order."""
    f, l = tab[qpos][:2], tab[qpos + T - 1][:2]
    out = []
    for t in range(lay.P):
        for tiles, s0, p0 in lay.runs((rank - t) % lay.P):
            out += [(s0 + u * T, p0 + u * T, class_from_bounds(f, l, p0 + u * T))
                    for u in interval(f[0], l[1], p0, tiles)]
    return out


def bwd_queries(lay, tab, rank, kpos):
    """dK/dV: query tiles of one key tile, reverse ring order."""
    f, l = tab[kpos][2:], tab[kpos + T - 1][2:]
    out = []
    for t in range(lay.P):
        for tiles, s0, p0 in lay.runs((rank + t) % lay.P):
            out += [(s0 + u * T, p0 + u * T, class_from_bounds(f, l, p0 + u * T))
                    for u in interval(f[0], l[1], p0, tiles)]
    return out


def query_tile_pairs(lay):
    """(rank, first slot, pos0, pos1) of the forward's items: two heads at one
    slot (even group) or two adjacent tiles of one rank (odd group)."""
    for slot in range(0, lay.S, T):
        rank = slot // lay.L
        p = lay.pos_of_slot(slot)
        yield rank, slot, p, p
        if (slot - rank * lay.L) % (2 * T) == 0:
            yield rank, slot, p, lay.pos_of_slot(slot + T)


def check_layout(S, P, zigzag, causal, window, cu):
    lay = Layout(S, P, zigzag)
    tab = bounds_table(S, causal, window, cu)
    vis = np.zeros((S, S), dtype=bool)
    for i in range(S):
        vis[i, tab[i][0]:tab[i][1] + 1] = True
    rng = random.Random(S + P)
    for i in rng.sample(range(S), min(S, 24)):
        for j in range(S):
            assert vis[i, j] == visible(S, causal, window, cu, i, j), (i, j)
    for f in range(4):
        col = [t[f] for t in tab]
        assert all(col[n] <= col[n + 1] for n in range(S - 1)), f
    for j in range(S):
        rows = np.nonzero(vis[:, j])[0]
        assert rows.min() == tab[j][2] and rows.max() == tab[j][3], j
    nt = S // T
    truth = np.array([[SKIP if not vis[a * T:(a + 1) * T, b * T:(b + 1) * T].any() else
                       FULL if vis[a * T:(a + 1) * T, b * T:(b + 1) * T].all() else MASK
                       for b in range(nt)] for a in range(nt)])
    for rank, slot, pos0, pos1 in query_tile_pairs(lay):
        need = {b * T for b in range(nt) if truth[pos0 // T, b] or truth[pos1 // T, b]}
        ring = fwd_ring(lay, tab, rank, pos0, pos1)
        kp = [p for _, p in ring]
        assert kp and len(set(kp)) == len(kp) and need <= set(kp)
        assert all(lay.pos_of_slot(s) == p for s, p in ring)
        for p in kp:  # the softmax's class of every visited tile
            assert class_from_bounds(tab[pos0][:2], tab[pos0 + T - 1][:2], p) == truth[pos0 // T, p // T]
        gathered = [p for _, p in fwd_gathered(lay, tab, pos0, pos1)]
        assert len(set(gathered)) == len(gathered) and need <= set(gathered)
        seen = []
        for owner in range(P):
            step = fwd_step(lay, tab, owner, pos0, pos1)
            block = {lay.pos_of_slot(owner * lay.L + u) for u in range(0, lay.L, T)}
            assert all(lay.pos_of_slot(owner * lay.L + s) == p for s, p in step)
            assert {p for _, p in step} <= block
            assert need & block <= {p for _, p in step}
            seen += [p for _, p in step]
        assert sorted(seen) == sorted(kp)  # the P steps visit what the ring visits
    for slot in range(0, S, T):
        rank, qp = slot // lay.L, lay.pos_of_slot(slot)
        seq = bwd_keys(lay, tab, rank, qp)
        assert all(lay.pos_of_slot(s) == p and c == truth[qp // T, p // T] for s, p, c in seq)
        assert sorted(p for _, p, _ in seq) == [b * T for b in range(nt) if truth[qp // T, b]]
    for kt in range(nt):
        kp = kt * T
        seq = bwd_queries(lay, tab, lay.slot_of_pos(kp) // lay.L, kp)
        assert all(lay.pos_of_slot(s) == p and c == truth[p // T, kt] for s, p, c in seq)
        assert sorted(p for _, p, _ in seq) == [a * T for a in range(nt) if truth[a, kt]]


LAYOUTS = [(1024, 4, True), (1024, 2, False), (2048, 8, True), (2048, 4, False),
           (1536, 3, True), (512, 1, True)]


@pytest.mark.parametrize("S,P,zigzag", LAYOUTS)
@pytest.mark.parametrize("causal,window", [(True, 0), (False, 0), (True, 1), (True, 129),
                                           (True, 300)])
def test_schedules_cover_exactly_the_visible_tiles(S, P, zigzag, causal, window):
    check_layout(S, P, zigzag, causal, window, None)


@pytest.mark.parametrize("S,P,zigzag", LAYOUTS[:4])
def test_schedules_with_packed_documents(S, P, zigzag):
    rng = random.Random(S * 7 + P)
    docsets = [[0, S], [0, 100, 101, 700, S], [0, 128, 256, 640, S], [0, 5, 5, S - 1, S]]
    docsets += [[0] + sorted(rng.sample(range(1, S), rng.randint(1, 10))) + [S] for _ in range(2)]
    for cu in docsets:
        for causal, window in [(True, 0), (False, 0), (True, 200)]:
            check_layout(S, P, zigzag, causal, window, cu)
