"""Model of the persistent decode kernel's mbarrier protocol, run on the CPU.

The kernel's three roles (producer warp: tile and operand copies; helper warp:
query state of each (b, h) segment, up to kAhead segments ahead, and the
finishing of middle segments; consumer warps: tiles, segment hand-off) wait on
barriers with parity waits.  Here each role is a generator that yields the
barrier phase it waits for; a random scheduler interleaves them.  Checked for
every partition of random ragged batches among CTAs, ring depths and slot
counts: no interleaving deadlocks, and no waiter ever falls two phases behind
a barrier (which a parity wait cannot tell from the phase it wants).

The ring sizes, slot counts and hand-off rules mirror decode.cu: S tile
stages, NBUF operand buffers, NQ query-state slots, two result slots; the
helper builds segment k only while k < done + kAhead (kAhead = NQ when q'
comes precomputed, 2 when the producer stages operands).  A model of the
protocol, not of the arithmetic: a change to the kernel's hand-off rules
must be mirrored here.
"""
import random

import pytest


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.phase = count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count


def segments_of(tiles):
    segs = []
    for bh in tiles:
        if not segs or segs[-1] != bh:
            segs.append(bh)
    return segs


def run(tiles, S, NBUF, NQ, qglobal, rng, kAhead=None):
    kAhead = kAhead or (NQ if qglobal else 2)
    full = [Bar(1) for _ in range(S)]
    empty = [Bar(8) for _ in range(S)]
    segfull, segempty = [Bar(1) for _ in range(2)], [Bar(1) for _ in range(2)]
    qready, qfree = [Bar(1) for _ in range(NQ)], [Bar(8) for _ in range(NQ)]
    resfull, resfree = [Bar(1) for _ in range(2)], [Bar(1) for _ in range(2)]
    nseg = len(segments_of(tiles))
    hazards = []

    def producer():
        issued = k = 0
        prev = None
        for bh in tiles:
            if not qglobal and bh != prev:
                if k >= NBUF:
                    yield segempty[k % NBUF], k // NBUF - 1
                segfull[k % NBUF].arrive()
                k += 1
                prev = bh
            s = issued % S
            if issued >= S:
                yield empty[s], issued // S - 1
            full[s].arrive()
            issued += 1

    def helper():
        built = done = 0
        more = True
        while True:
            while more and built < done + kAhead:
                if built >= nseg:
                    more = False
                    break
                k = built
                if not qglobal:
                    yield segfull[k % NBUF], k // NBUF
                if k >= NQ:
                    yield qfree[k % NQ], k // NQ - 1
                if not qglobal:
                    segempty[k % NBUF].arrive()
                qready[k % NQ].arrive()
                built += 1
            if done == built or (not more and done == built - 1):
                return  # the consumers finish the CTA's last segment
            yield resfull[done & 1], done // 2
            resfree[done & 1].arrive()
            done += 1

    def consumers():
        k = i = 0
        prev = None
        for bh in tiles:
            if bh != prev:
                if prev is not None:  # hand segment k - 1 to the helper
                    j = k - 1
                    if j >= 2:
                        yield resfree[j & 1], j // 2 - 1
                    resfull[j & 1].arrive()
                yield qready[k % NQ], k // NQ
                for _ in range(8):
                    qfree[k % NQ].arrive()
                k += 1
                prev = bh
            s = i % S
            yield full[s], i // S
            for _ in range(8):
                empty[s].arrive()
            i += 1

    roles = [producer(), helper(), consumers()]
    waiting = [next(g, None) for g in roles]
    while any(w is not None for w in waiting):
        ready = [r for r, w in enumerate(waiting) if w is not None and w[0].phase > w[1]]
        for r, w in enumerate(waiting):
            if w is not None and w[0].phase > w[1] + 1:
                hazards.append(r)
        if not ready:
            return False, hazards
        r = rng.choice(ready)
        waiting[r] = next(roles[r], None)
    return True, hazards


def cta_tiles(lens, H, T, C, c):
    """The (b, h) of every tile CTA c owns: the flattened (b, h, tile) space
    split evenly over CW = min(C, G) CTAs, as in the kernel's split plan."""
    tiles_b = [(n + T - 1) // T for n in lens]
    pre = [0]
    for t in tiles_b:
        pre.append(pre[-1] + t)
    G = H * pre[-1]
    CW = min(C, G)
    if c >= CW:
        return []
    out = []
    for g in range(G * c // CW, G * (c + 1) // CW):
        b = max(i for i in range(len(lens)) if H * pre[i] <= g)
        out.append((b, (g - H * pre[b]) // tiles_b[b]))
    return out


@pytest.mark.parametrize("qglobal", [True, False])
def test_no_deadlock_or_phase_aliasing(qglobal):
    rng = random.Random(11 if qglobal else 12)
    runs = 0
    for _ in range(60):
        B = rng.randint(1, 24)
        H = rng.choice([1, 2, 4, 32])
        T = rng.choice([64, 512, 1024])
        lens = [rng.randint(0, 4096) for _ in range(B)]
        C = rng.choice([296, 100, 37, 8, 3])
        for c in rng.sample(range(C), min(C, 6)):
            tiles = cta_tiles(lens, H, T, C, c)
            if not tiles:
                continue
            for S, NBUF, NQ in ((4, 2, 4), (2, 1, 4), (3, 2, 2), (8, 2, 4), (2, 2, 2)):
                ok, hazards = run(tiles, S, NBUF, NQ, qglobal, rng)
                runs += 1
                assert ok, (segments_of(tiles), S, NBUF, NQ)
                assert not hazards, (segments_of(tiles), S, NBUF, NQ)
    assert runs > 200


def test_model_catches_a_helper_that_runs_too_far_ahead():
    """The check is not vacuous: a helper allowed 2 * NQ segments ahead (it then
    waits for a query slot the consumers cannot free before it finishes an
    older segment) deadlocks on some partitions."""
    rng = random.Random(5)
    bad = 0
    for _ in range(40):
        B = rng.randint(1, 24)
        lens = [rng.randint(0, 4096) for _ in range(B)]
        for c in range(3):
            tiles = cta_tiles(lens, 32, 64, 37, c)
            if tiles:
                ok, hazards = run(tiles, 2, 1, 4, True, rng, kAhead=8)
                bad += (not ok) or bool(hazards)
    assert bad > 0
