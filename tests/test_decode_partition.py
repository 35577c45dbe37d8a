"""The decode kernel's stream-K work split, modelled on the CPU and checked for the
invariants its merge relies on, over random length mixes, head counts and grid sizes.

Units are 16-token blocks of one (sequence, kv-head group), numbered sequence-major; CTA c
takes units [c*U, (c+1)*U) with U = ceil(total / CTAs).  A segment (one sequence's units of
one kv-head group) that a CTA covers whole is written directly; otherwise every covering CTA
writes a partial state to slot heads_per_unit * (segment + c) + head, and the CTA of the
segment's first interior boundary merges it.  Checked: every unit is covered exactly once;
each split segment gets exactly one partial per covering CTA and exactly one merging CTA;
partial slots never collide and fit the workspace of B*Hkv + 2*CTAs slots.

The tensor-core decode splits by cost instead: a unit costs 1 and a segment's first unit 3
more, CTA c starts at the first unit whose running cost key(u) * CTAs reaches c * total cost
(equal counts when the problem is too small for every CTA to get a unit).  Its closed form is
checked against a brute-force walk over every unit, and the same invariants are checked for
its CTA ranges, with the merge's owner found by searching the CTAs' first units."""
import math

import numpy as np
import pytest


def _owner(starts, nctas, u):
    """The last CTA c < nctas whose first unit is at or before u."""
    return int(np.searchsorted(np.asarray(starts[:nctas]), u, side="right") - 1)


def _model(blocks, hkv, hpu, nctas, starts=None):
    hu = hkv // hpu
    pfx = np.concatenate([[0], np.cumsum(blocks)])
    total = hu * int(pfx[-1])
    U = max(1, math.ceil(total / nctas)) if total else 1
    if starts is None:
        starts = [min(c * U, total) for c in range(nctas)] + [total]
    writes = {}      # slot -> (segment, cta, head)
    whole = set()
    covered = np.zeros(total, np.int32)
    for c in range(nctas):
        u0, u1 = starts[c], starts[c + 1]
        if u0 >= u1:
            continue
        covered[u0:u1] += 1
        u = u0
        while u < u1:
            b = int(np.searchsorted(hu * pfx, u, side="right") - 1)
            while b + 1 < len(blocks) and blocks[b] == 0 and hu * pfx[b + 1] <= u:
                b += 1
            nb = int(blocks[b])
            rel = u - hu * int(pfx[b])
            kvg, blk = rel // nb, rel % nb
            piece = min(nb - blk, u1 - u)
            segu = b * hu + kvg
            if blk == 0 and piece == nb:
                whole.add(segu)
            else:
                for hd in range(hpu):
                    slot = hpu * (segu + c) + hd
                    assert slot not in writes, "partial slots collide"
                    assert slot < len(blocks) * hkv + 2 * nctas, "slot outside the workspace"
                    writes[slot] = (segu, c, hd)
            u += piece
    # the merging CTA of every split segment (the combine kernel's rule)
    merged = {}
    for c in range(1, nctas):
        x = starts[c]
        if x >= total:
            continue
        b = int(np.searchsorted(hu * pfx, x, side="right") - 1)
        nb = int(pfx[b + 1] - pfx[b])
        kvg = (x - hu * int(pfx[b])) // nb
        start = hu * int(pfx[b]) + kvg * nb
        if start == x:
            continue
        c0, c1 = _owner(starts, nctas, start), _owner(starts, nctas, start + nb - 1)
        if c0 != c - 1:
            continue
        segu = b * hu + kvg
        assert segu not in merged, "segment merged twice"
        merged[segu] = (c0, c1)
    return total, covered, writes, whole, merged, starts, hu, pfx


UNIT_COST, PIECE_COST = 1, 3


def _cost_starts(tiles, hu, nctas):
    """The cost-balanced CTA starts in closed form: the sequence whose keys reach the
    threshold by bisection on its prefix sums, then the kv head and tile by division."""
    tiles = np.asarray(tiles, np.int64)
    B = len(tiles)
    pfx = np.concatenate([[0], np.cumsum(tiles)])
    ne = np.concatenate([[0], np.cumsum(tiles > 0)])
    total = hu * int(pfx[-1])
    ctot = UNIT_COST * total + PIECE_COST * hu * int(ne[-1])
    U = (total + nctas - 1) // nctas if total else 1
    by_cost = ctot >= (UNIT_COST + PIECE_COST) * nctas

    def base(b):
        return hu * (UNIT_COST * int(pfx[b]) + PIECE_COST * int(ne[b]))

    def unit_at(thr):
        lo, hi = 0, B - 1
        while lo < hi:
            mid = (lo + hi) // 2
            if base(mid + 1) >= thr + UNIT_COST:
                hi = mid
            else:
                lo = mid + 1
        nt = int(tiles[lo])
        u = hu * int(pfx[lo])
        r = thr - (base(lo) + PIECE_COST)
        if r > 0:
            seg = UNIT_COST * nt + PIECE_COST
            kvh, rem = divmod(r, seg)
            tile = 0
            if rem > 0:
                if rem <= UNIT_COST * (nt - 1):
                    tile = -(-rem // UNIT_COST)
                else:
                    kvh += 1
            u += kvh * nt + tile
        return u

    starts = []
    for c in range(nctas + 1):
        if c == 0:
            starts.append(0)
        elif c == nctas:
            starts.append(total)
        elif by_cost:
            starts.append(unit_at((c * ctot + nctas - 1) // nctas))
        else:
            starts.append(min(c * U, total))
    return starts, by_cost, ctot


def _keys(tiles, hu):
    """key(u) of every unit by walking them: UNIT_COST per unit before u, PIECE_COST per
    segment start at or before u."""
    keys, starts_seen, u = [], 0, 0
    for nt in tiles:
        for _ in range(hu):
            for t in range(int(nt)):
                if t == 0:
                    starts_seen += 1
                keys.append(UNIT_COST * u + PIECE_COST * starts_seen)
                u += 1
    return np.asarray(keys, np.int64)


def _lengths(g, B):
    L = g.integers(0, 3000, B)
    L[g.random(B) < 0.2] = 0                                   # some empty sequences
    short = g.random(B) < 0.3
    L[short] = g.integers(1, 200, int(short.sum()))            # many one-piece sequences
    return L


@pytest.mark.parametrize("seed", range(40))
def test_cost_split_matches_brute_force_and_balances(seed):
    g = np.random.default_rng(1000 + seed)
    B = int(g.integers(1, 60))
    tiles = (_lengths(g, B) + 127) // 128
    hu = int(g.choice([1, 2, 4, 8]))
    nctas = int(g.choice([1, 3, 7, 148]))
    starts, by_cost, ctot = _cost_starts(tiles, hu, nctas)
    total = hu * int(tiles.sum())
    assert starts[0] == 0 and starts[-1] == total and all(a <= b for a, b in zip(starts, starts[1:]))
    if not by_cost:
        return
    keys = _keys(tiles, hu)
    assert len(keys) == total and ctot == UNIT_COST * total + PIECE_COST * hu * int((tiles > 0).sum())
    for c in range(1, nctas):
        want = int(np.argmax(keys * nctas >= c * ctot))       # the first unit reaching c's share
        assert starts[c] == want, (c, starts[c], want)
    # every CTA gets a unit, and no CTA's cost exceeds its share by more than one unit's
    cost = np.diff(np.concatenate([keys, [ctot]])) if total else np.zeros(0)
    for c in range(nctas):
        u0, u1 = starts[c], starts[c + 1]
        assert u1 > u0
        assert int(cost[u0:u1].sum()) <= -(-ctot // nctas) + UNIT_COST + PIECE_COST


@pytest.mark.parametrize("seed", range(40))
def test_cost_split_merge_invariants(seed):
    g = np.random.default_rng(2000 + seed)
    B = int(g.integers(1, 60))
    tiles = (_lengths(g, B) + 127) // 128
    hkv = int(g.choice([1, 2, 4, 8]))
    nctas = int(g.choice([1, 3, 7, 148]))
    starts, _, _ = _cost_starts(tiles, hkv, nctas)
    total, covered, writes, whole, merged, starts, hu, pfx = _model(tiles, hkv, 1, nctas, starts)
    assert np.all(covered == 1)
    for segu in range(B * hu):
        b, k = divmod(segu, hu)
        nb = int(tiles[b])
        if nb == 0:
            continue
        start = hu * int(pfx[b]) + k * nb
        c0, c1 = _owner(starts, nctas, start), _owner(starts, nctas, start + nb - 1)
        if segu in whole:
            assert c0 == c1 and segu not in merged
        else:
            assert merged.get(segu) == (c0, c1)
            for c in range(c0, c1 + 1):
                assert writes.get(segu + c) == (segu, c, 0)
    # the CTAs' first units sit in the first slot past those the split can use
    assert max(writes, default=-1) < B * hkv + nctas


@pytest.mark.parametrize("seed", range(40))
def test_partition_invariants(seed):
    g = np.random.default_rng(seed)
    B = int(g.integers(1, 40))
    L = g.integers(0, 3000, B)
    L[g.random(B) < 0.2] = 0                                   # some empty sequences
    blocks = (L + 15) // 16
    hkv = int(g.choice([1, 2, 4, 8]))
    hpu = 2 if hkv % 2 == 0 and g.random() < 0.5 else 1
    nctas = int(g.choice([1, 3, 7, 148, 444, 592]))
    total, covered, writes, whole, merged, starts, hu, pfx = _model(blocks, hkv, hpu, nctas)
    assert np.all(covered == 1)
    segs = [(b * hu + k, int(blocks[b])) for b in range(B) for k in range(hu) if blocks[b] > 0]
    for segu, nb in segs:
        b, k = divmod(segu, hu)
        start = hu * int(pfx[b]) + k * nb
        c0, c1 = _owner(starts, nctas, start), _owner(starts, nctas, start + nb - 1)
        if segu in whole:
            assert c0 == c1 and segu not in merged
        else:
            assert merged.get(segu) == (c0, c1), "split segment without exactly one merge"
            for c in range(c0, c1 + 1):
                for hd in range(hpu):
                    assert writes.get(hpu * (segu + c) + hd) == (segu, c, hd)
    assert len(writes) == sum((c1 - c0 + 1) * hpu for (c0, c1) in merged.values())
