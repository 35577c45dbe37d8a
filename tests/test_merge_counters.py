"""The tensor-core decode merges a segment that several CTAs cut in the kernel: each CTA adds
one arrival to a counter and the last to arrive merges.  The plain decode's workspace is
not zeroed, so its counters carry a per-launch tag in their high 48 bits: an arrival that
finds another tag (left by an earlier launch, an aborted one, or whatever the memory held)
restarts the count at 1, and the last arriver resets the counter to 0.  This models that
protocol (the compare-and-swap loop of tc_arrive_epoch in csrc/decode_tc.cu) on the CPU and
checks what the merge relies on, over random interleavings and initial contents."""
import random

import pytest

MASK64 = (1 << 64) - 1


def arrive(mem, i, tag):
    """One arrival, as the device does it: read, then compare-and-swap until it sticks.
    Returns the count after this arrival (this one included)."""
    cur = mem[i]
    while True:
        nv = (cur + 1) & MASK64 if (cur >> 16) == tag else ((tag << 16) | 1)
        if mem[i] == cur:          # the compare-and-swap succeeds
            mem[i] = nv
            return nv & 0xFFFF
        cur = mem[i]               # it failed: retry with the value seen


def run_launch(mem, tag, segs, rng):
    """segs: {counter index: number of CTAs cutting that segment}.  Arrivals of different
    segments interleave at random; returns how many merges each segment got."""
    pending = [(i, n) for i, n in segs.items() for _ in range(n)]
    rng.shuffle(pending)
    merges = {i: 0 for i in segs}
    for i, n in pending:
        if arrive(mem, i, tag) == n:
            merges[i] += 1
            mem[i] = 0             # the merging CTA resets its counter
    return merges


@pytest.mark.parametrize("seed", range(50))
def test_every_split_segment_merges_exactly_once(seed):
    rng = random.Random(seed)
    n = 148
    mem = [rng.getrandbits(64) for _ in range(n)]     # whatever the workspace held
    tag = rng.getrandbits(47) | 1                     # per-process start, never 0
    for launch in range(4):
        segs = {i: rng.randint(2, 5) for i in rng.sample(range(n), rng.randint(1, 40))}
        # an arbitrary leftover may carry this very tag only with probability 2^-48; a
        # counter left by an aborted launch of an OLDER tag must not disturb this one
        merges = run_launch(mem, tag + launch, segs, rng)
        assert all(m == 1 for m in merges.values()), merges
        assert all(mem[i] == 0 for i in segs)


def test_replayed_tag_starts_clean():
    """A captured graph replays the same tag: the reset to 0 by the last arriver is what
    makes the second replay count from 1 again."""
    rng = random.Random(7)
    mem = [0] * 8
    for _ in range(3):
        merges = run_launch(mem, 12345, {3: 4, 5: 2}, rng)
        assert merges == {3: 1, 5: 1}


def test_leftover_count_of_another_tag_is_replaced():
    mem = [(99 << 16) | 3]         # an earlier launch's count that never finished
    assert arrive(mem, 0, 100) == 1
    assert arrive(mem, 0, 100) == 2
