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
stages, NBUF operand buffers, NQ query-state slots, two result slots, and a
queue of kSegQ segment descriptors through which the producer hands each
segment (a run of tiles of one (b, h): a piece of the CTA's static range, or a
chunk it claimed) to the helper and the consumers, followed by an end marker;
a queue slot is reused once the helper and all eight consumer warps have read
it.  The consumers read the next descriptor before handing a segment over, and
finish the CTA's last segment themselves.  The helper builds segment k only
while k < done + kAhead (kAhead = NQ when q' comes precomputed, 2 when the
producer stages operands).  A model of the protocol, not of the arithmetic: a
change to the kernel's hand-off rules must be mirrored here.
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
    """Tile counts of the runs of equal (b, h) in a CTA's tile list."""
    segs = []
    prev = None
    for bh in tiles:
        if bh != prev:
            segs.append(0)
            prev = bh
        segs[-1] += 1
    return segs


def run(segs, S, NBUF, NQ, qglobal, rng, kAhead=None, Q=4, helper_frees=True):
    kAhead = kAhead or (NQ if qglobal else 2)
    full = [Bar(1) for _ in range(S)]
    empty = [Bar(8) for _ in range(S)]
    segfull, segempty = [Bar(1) for _ in range(2)], [Bar(1) for _ in range(2)]
    qready, qfree = [Bar(1) for _ in range(NQ)], [Bar(8) for _ in range(NQ)]
    resfull, resfree = [Bar(1) for _ in range(2)], [Bar(1) for _ in range(2)]
    sqfull, sqfree = [Bar(1) for _ in range(Q)], [Bar(9 if helper_frees else 8) for _ in range(Q)]
    queue = list(segs) + [0]  # descriptors in emission order; 0 tiles ends the queue
    hazards = []

    def producer():
        issued = k = 0
        for n, nt in enumerate(queue):
            if n >= Q:  # queue slot free: read by the helper and the eight consumer warps
                yield sqfree[n % Q], n // Q - 1
            sqfull[n % Q].arrive()
            if nt == 0:
                return
            if not qglobal:
                if k >= NBUF:
                    yield segempty[k % NBUF], k // NBUF - 1
                segfull[k % NBUF].arrive()
                k += 1
            for _ in range(nt):
                s = issued % S
                if issued >= S:
                    yield empty[s], issued // S - 1
                full[s].arrive()
                issued += 1

    def helper():
        built = done = nread = 0
        more = True
        while True:
            while more and built < done + kAhead:
                yield sqfull[nread % Q], nread // Q
                if helper_frees:
                    sqfree[nread % Q].arrive()
                nt = queue[nread]
                nread += 1
                if nt == 0:
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
        k = i = nread = 0

        def read():
            nonlocal nread
            yield sqfull[nread % Q], nread // Q
            for _ in range(8):
                sqfree[nread % Q].arrive()
            nread += 1

        yield from read()
        nt = queue[0]
        while nt > 0:
            yield qready[k % NQ], k // NQ
            for _ in range(8):
                qfree[k % NQ].arrive()
            k += 1
            for _ in range(nt):
                s = i % S
                yield full[s], i // S
                for _ in range(8):
                    empty[s].arrive()
                i += 1
            yield from read()
            nxt = queue[nread - 1]
            if nxt == 0:
                return  # finish the last segment here
            j = k - 1  # hand segment k - 1 to the helper
            if j >= 2:
                yield resfree[j & 1], j // 2 - 1
            resfull[j & 1].arrive()
            nt = nxt

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
    """Static plan: every CTA's range of the flattened (b, h, tile) space."""
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
                ok, hazards = run(segments_of(tiles), S, NBUF, NQ, qglobal, rng)
                runs += 1
                assert ok, (segments_of(tiles), S, NBUF, NQ)
                assert not hazards, (segments_of(tiles), S, NBUF, NQ)
    assert runs > 200


@pytest.mark.parametrize("qglobal", [True, False])
def test_dynamic_chunks_no_deadlock_or_phase_aliasing(qglobal):
    """Dynamic plan: a CTA claims any number of chunks (none included) of one
    to a few tiles each, in any order of heads."""
    rng = random.Random(21 if qglobal else 22)
    for _ in range(400):
        segs = [rng.randint(1, 4) for _ in range(rng.choice([0, 1, 2, 3, 5, 9, 17]))]
        S, NBUF, NQ = rng.choice(((4, 2, 4), (2, 1, 4), (3, 2, 2), (8, 2, 4), (2, 2, 2)))
        ok, hazards = run(segs, S, NBUF, NQ, qglobal, rng)
        assert ok and not hazards, (segs, S, NBUF, NQ)


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
                ok, hazards = run(segments_of(tiles), 2, 1, 4, True, rng, kAhead=8, Q=16)
                bad += (not ok) or bool(hazards)
    assert bad > 0


def test_model_catches_a_queue_slot_freed_without_the_helper():
    """The check is not vacuous for the descriptor queue either: if a slot were
    reused once the consumers alone had read it, the helper (which reads
    descriptors only as far as kAhead allows) falls a full queue cycle behind
    on some schedules."""
    rng = random.Random(9)
    bad = 0
    for _ in range(300):
        segs = [rng.randint(1, 3) for _ in range(rng.randint(6, 17))]
        ok, hazards = run(segs, 4, 2, 2, True, rng, helper_frees=False)
        bad += (not ok) or bool(hazards)
    assert bad > 0
