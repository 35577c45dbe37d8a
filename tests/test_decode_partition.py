"""The decode kernel's stream-K work split, modelled on the CPU and checked for the
invariants its merge relies on, over random length mixes, head counts and grid sizes.

Units are 16-token blocks of one (sequence, kv-head group), numbered sequence-major; CTA c
takes units [c*U, (c+1)*U) with U = ceil(total / CTAs).  A segment (one sequence's units of
one kv-head group) that a CTA covers whole is written directly; otherwise every covering CTA
writes a partial state to slot heads_per_unit * (segment + c) + head, and the CTA of the
segment's first interior boundary merges it.  Checked: every unit is covered exactly once;
each split segment gets exactly one partial per covering CTA and exactly one merging CTA;
partial slots never collide and fit the workspace of B*Hkv + 2*CTAs slots."""
import math

import numpy as np
import pytest


def _model(blocks, hkv, hpu, nctas):
    hu = hkv // hpu
    pfx = np.concatenate([[0], np.cumsum(blocks)])
    total = hu * int(pfx[-1])
    U = max(1, math.ceil(total / nctas)) if total else 1
    writes = {}      # slot -> (segment, cta, head)
    whole = set()
    covered = np.zeros(total, np.int32)
    for c in range(nctas):
        u0, u1 = c * U, min((c + 1) * U, total)
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
        x = c * U
        if x >= total:
            continue
        b = int(np.searchsorted(hu * pfx, x, side="right") - 1)
        nb = int(pfx[b + 1] - pfx[b])
        kvg = (x - hu * int(pfx[b])) // nb
        start = hu * int(pfx[b]) + kvg * nb
        if start == x:
            continue
        c0, c1 = start // U, (start + nb - 1) // U
        if c0 != c - 1:
            continue
        segu = b * hu + kvg
        assert segu not in merged, "segment merged twice"
        merged[segu] = (c0, c1)
    return total, covered, writes, whole, merged, U, hu, pfx


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
    total, covered, writes, whole, merged, U, hu, pfx = _model(blocks, hkv, hpu, nctas)
    assert np.all(covered == 1)
    segs = [(b * hu + k, int(blocks[b])) for b in range(B) for k in range(hu) if blocks[b] > 0]
    for segu, nb in segs:
        b, k = divmod(segu, hu)
        start = hu * int(pfx[b]) + k * nb
        c0, c1 = start // U, (start + nb - 1) // U
        if segu in whole:
            assert c0 == c1 and segu not in merged
        else:
            assert merged.get(segu) == (c0, c1), "split segment without exactly one merge"
            for c in range(c0, c1 + 1):
                for hd in range(hpu):
                    assert writes.get(hpu * (segu + c) + hd) == (segu, c, hd)
    assert len(writes) == sum((c1 - c0 + 1) * hpu for (c0, c1) in merged.values())
