"""Model of the one-kernel step's barrier and copy accounting, run on the CPU.

Every barrier of `step_cluster_kernel` is initialised with one arrival and
waited for once (parity 0).  A phase completes only when its arrival is made
and the transaction bytes it expects have all landed; a mismatch would leave
a waiter to its one-second bound.  This model restates, for every rank of a
cluster, which barriers receive an arrive / expect_tx and which copies or
st.async stores complete bytes on them. For a grid of shapes and lengths
(new row at every kind of position, a full cache, an invalid length, int8
weights, one- to eight-CTA clusters) it checks that:
  * each barrier somebody waits for gets exactly its one arrival, and
    delivered bytes == expected bytes;
  * every bulk copy is a multiple of 16 bytes at a 16-byte-aligned offset, and
    fits its shared-memory region;
  * st.async partial rows from different ranks land in disjoint slots;
  * the owner and the merging rank are consistent with the chunking.
A model of the protocol, not of the arithmetic: a change to the kernel's copy
plan must be mirrored here.
"""
import itertools

import pytest

T = 256                 # tokens per tile (one token per lane, 256 consumer threads)
CHUNKS = 4              # A slice chunks per unit
APPEND_WARPS = 8


def chunk_of(L_cap, cs):
    return ((L_cap + cs - 1) // cs + 7) & ~7


class Barrier:
    def __init__(self):
        self.arrivals, self.expected, self.delivered = 0, 0, 0

    def arrive(self, tx=0):
        self.arrivals += 1
        self.expected += tx

    def complete(self, nbytes):
        self.delivered += nbytes

    def done(self):
        return self.arrivals == 1 and self.expected == self.delivered


def copy(bar, nbytes, offset, region):
    assert nbytes % 16 == 0 and offset % 16 == 0, (nbytes, offset)
    assert offset + nbytes <= region, (offset, nbytes, region)
    bar.complete(nbytes)


def model(cs, L_cap, pos, E, r, Hd, rb, w8):
    """Run the copy plan of every rank of one cluster; return the checks' inputs."""
    W = r
    chunk = chunk_of(L_cap, cs)
    assert chunk <= T  # the host launches the kernel only then
    ok = 0 <= pos < L_cap
    lead = pos // chunk if ok else 0
    assert lead < cs
    Ec = E // cs
    slice_bytes = Ec * r * (1 if w8 else 2)
    piece = slice_bytes // CHUNKS
    bb, qb, sb = W * Hd * (1 if w8 else 2), Hd * 2, (Hd * 4 if w8 else 0)
    seg_region = (W * Hd * 2 + Hd * 2 + 127) // 128 * 128
    bvs_region = W * Hd * 2
    code_bytes, scale_bytes = T * rb, T * 2
    ranks = []
    for rank in range(cs):
        lo = min(L_cap, rank * chunk)
        hi = min(L_cap, lo + chunk)
        len_old = pos if ok else (pos if 0 <= pos <= L_cap else 0)
        n_old = max(0, min(hi, len_old) - lo)
        own = ok and rank == lead
        bars = {k: Barrier() for k in ("full", "segfull", "bvs", "parts", "rows", "pos")}
        bars.update({("a", u, c): Barrier() for u in range(2) for c in range(CHUNKS)})
        # producer lane
        bars["segfull"].arrive(bb + qb + sb)
        copy(bars["segfull"], bb, 0, seg_region)
        if w8:
            copy(bars["segfull"], sb, bb + qb, seg_region)
        copy(bars["segfull"], qb, bb, seg_region)
        for u in range(2):
            for c in range(CHUNKS):
                bars[("a", u, c)].arrive(piece)
                copy(bars[("a", u, c)], piece, c * piece, slice_bytes)
        if rank == lead and cs > 1:
            if ok:
                bars["rows"].arrive((cs - 1) * 2 * r * 4)
            bars["parts"].arrive((cs - 1) * (W + 2) * 4)
        bars["pos"].arrive()
        if rank == lead:
            bars["bvs"].arrive(bb + sb)
            for off in range(0, bb, 32768):
                copy(bars["bvs"], min(32768, bb - off), off, bvs_region)
            if w8:
                copy(bars["bvs"], sb, bb, bvs_region)
        if n_old > 0:
            cbytes, sbytes = n_old * rb, ((n_old + 7) & ~7) * 2
            assert n_old <= T and sbytes <= scale_bytes
            bars["full"].arrive(2 * cbytes + 2 * sbytes)
            copy(bars["full"], cbytes, 0, code_bytes)
            copy(bars["full"], cbytes, code_bytes, 2 * code_bytes)
            copy(bars["full"], sbytes, 2 * code_bytes, 2 * code_bytes + scale_bytes)
            copy(bars["full"], sbytes, 2 * code_bytes + scale_bytes, 2 * code_bytes + 2 * scale_bytes)
            # the scale copies read rows [lo, lo + ceil8(n_old)): inside the cache
            assert lo + ((n_old + 7) & ~7) <= L_cap
        else:
            bars["full"].arrive()
        if own:
            assert lo <= pos < hi and pos - lo < T  # the new row's slot in the staged tile
        ranks.append(dict(rank=rank, lo=lo, hi=hi, n_old=n_old, own=own, bars=bars))
    # st.async partial rows: K and V append partials to the owner, decode partials to the merging rank
    rows_into, parts_into = {}, {}
    for R in ranks:
        if ok and R["rank"] != lead:
            slots = range(R["rank"] * 2 * r, (R["rank"] + 1) * 2 * r)  # reduce over nb = 2 rows of r
            for j in slots:
                assert j not in rows_into
                rows_into[j] = R["rank"]
            ranks[lead]["bars"]["rows"].complete(2 * r * 4)
        if R["rank"] != lead:
            for j in range(R["rank"] * (W + 2), (R["rank"] + 1) * (W + 2)):
                assert j not in parts_into
                parts_into[j] = R["rank"]
            ranks[lead]["bars"]["parts"].complete((W + 2) * 4)
    return ok, lead, ranks


def waited(ok, lead, cs, R):
    """The barriers some thread of this rank waits for."""
    w = ["segfull", "pos", "full"] + [("a", u, c) for u in range(2) for c in range(CHUNKS)]
    if R["rank"] == lead:
        w.append("bvs")
        if cs > 1:
            w.append("parts")
    if R["own"] and cs > 1:
        w.append("rows")
    return w


SHAPES = [  # (cs, L_cap, E, r, Hd, rowbytes)
    (8, 1600, 4096, 32, 128, 32), (8, 1608, 4096, 32, 128, 32), (8, 1024, 2048, 32, 128, 16),
    (2, 256, 512, 32, 64, 32), (1, 128, 256, 32, 64, 32), (4, 1024, 1024, 32, 128, 32),
]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("w8", [False, True])
def test_every_wait_completes_and_copies_fit(shape, w8):
    cs, L_cap, E, r, Hd, rb = shape
    chunk = chunk_of(L_cap, cs)
    positions = sorted({0, 1, 7, 8, chunk - 1, chunk, chunk + 1, L_cap // 2, L_cap - 2, L_cap - 1, L_cap, L_cap + 5,
                        -1} & set(range(-1, L_cap + 6)))
    for pos in positions:
        ok, lead, ranks = model(cs, L_cap, pos, E, r, Hd, rb, w8)
        assert sum(R["own"] for R in ranks) == (1 if ok else 0)
        for R in ranks:
            for name in waited(ok, lead, cs, R):
                assert R["bars"][name].done(), (shape, w8, pos, R["rank"], name, vars(R["bars"][name]))


def test_old_rows_are_the_rows_below_the_new_one():
    """Each rank stages exactly the rows of its chunk below the new row (or below
    the unchanged length when nothing is appended), and the chunks tile [0, L_cap)."""
    for cs, L_cap in itertools.product([1, 2, 4, 8], [8, 128, 256, 1000, 1600, 2048]):
        chunk = chunk_of(L_cap, cs)
        if chunk > T:
            continue
        for pos in (0, 5, chunk, L_cap - 1, L_cap):
            _, _, ranks = model(cs, L_cap, pos, 4096 if cs > 1 else 256, 32, 128, 32, False)
            covered = [i for R in ranks for i in range(R["lo"], R["hi"])]
            assert covered == list(range(L_cap))
            below = min(pos, L_cap)
            assert sum(R["n_old"] for R in ranks) == below
