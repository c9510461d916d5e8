"""Deadlock check of the paired-row backward's schedule (two CTAs of a cluster), on the CPU.

Each CTA runs a cross-tile pipeline over its own 4-slot ring (the next tile's 14 S / dP
items interleaved as whole (K, Q, dO) triples, one triple after each of gradient blocks
4..8, so a key chunk is never held across a gradient block's loads) with its own
gradient blocks: dQ~ 0-4 (one chunk each), then the key-side blocks over both rows (rank 0
dV 0-3, rank 1 dK~ 0-4; two chunks each: the own row's, then the partner's).  The CTAs are
coupled through the exchanged P / dS tile:
  * softmax of tile i starts when its S / dP are formed and its own gradient MMAs of tile
    i - 1 completed; at its start it grants the partner the copy of tile i (remote arrive),
    then (i >= 1) waits for the partner's grant before writing its copy source; when the
    tile is written it issues the copy into the partner's buffer;
  * the MMA warp reads the partner's tile from the second half of the first key-side block
    on, after the partner's copy of that tile was issued.
The model replays both CTAs against these dependencies and the ring / staging / row-id
rules of the single-row model and checks that every role of both CTAs finishes.
"""
import pytest

def group_items(g):
    """S / dP items of group g: (K_g, Q_g, dO_g), the last group (K4, Q4)."""
    return [j for j in range(3 * g, 3 * g + 3) if j < 14]


def nblocks(rank):
    return 10 if rank else 9


def sdp_item(j):
    c = j // 3
    return j - 3 * c, c


INTER = 4  # first gradient block followed by a group (the same on both ranks)


def schedule(rank, ntiles):
    """Events (tile, kind, index, half) in issue order: ("S", j, 0) and ("G", k, h)."""
    nb = nblocks(rank)
    inter = INTER
    ev = [(0, "S", j, 0) for j in range(14)]
    for i in range(ntiles):
        for k in range(nb):
            for h in range(1 if k < 5 else 2):
                ev.append((i, "G", k, h))
            if i + 1 < ntiles and k >= inter:
                ev += [(i + 1, "S", j, 0) for j in group_items(k - inter)]
    return ev


def release_points(ev):
    rel = {}
    for idx, (i, typ, x, h) in enumerate(ev):
        if typ == "G":
            rel[idx] = idx
            continue
        kind, c = sdp_item(x)
        if kind != 0:
            rel[idx] = idx
        if kind == 2 or c == 4:
            kidx = max(e for e in range(idx + 1) if ev[e][:3] == (i, "S", 3 * c))
            rel[kidx] = idx
    return rel


class Cta:
    def __init__(self, rank, ntiles, slots):
        self.rank, self.nt, self.slots = rank, ntiles, slots
        self.ev = schedule(rank, ntiles)
        self.rel = release_points(self.ev)
        self.nb = nblocks(rank)
        self.loaded = self.issued = self.flushed = 0
        self.freed = set()
        self.staged = 0
        self.started = -1     # last tile whose softmax started (grant sent)
        self.written = -1     # last tile whose P / dS are written and copy issued
        self.sdp_done = -1
        self.grad_done = -1
        self.blocks = 0
        self.tiles_flushed = 0

    def done(self):
        n = len(self.ev)
        return (self.loaded == n and self.issued == n and self.flushed == self.nb * self.nt
                and self.written == self.nt - 1)


def step(c, peer, grant_before_wait=True):
    progress = False
    n = len(c.ev)
    if c.loaded < n:  # producer
        i, typ, x, h = c.ev[c.loaded]
        ready = True
        if typ == "S" and x == 0 and c.staged <= i:
            if c.tiles_flushed < i - 1:
                ready = False
            else:
                c.staged = i + 1
        if ready and c.loaded >= c.slots and (c.loaded - c.slots) not in c.freed:
            ready = False
        if ready:
            c.loaded += 1
            progress = True
    if c.issued < c.loaded:  # MMA
        i, typ, x, h = c.ev[c.issued]
        ready = True
        if typ == "G" and h == 0:
            if x == 0 and c.written < i:
                ready = False
            if c.blocks >= 2 and c.flushed < c.blocks - 1:
                ready = False
        if typ == "G" and x == 5 and h == 1 and peer.written < i:  # the partner's copy of tile i
            ready = False
        if ready:
            if typ == "G":
                if h == 0:
                    c.blocks += 1
                last_half = 0 if x < 5 else 1
                if x == c.nb - 1 and h == last_half:
                    c.grad_done = i
            elif x == 13:
                c.sdp_done = i
            c.freed.update(k for k, r in c.rel.items() if r == c.issued)
            c.issued += 1
            progress = True
    t = c.started + 1  # softmax start: grant the partner's copy of tile t
    if t < c.nt and c.sdp_done >= t and c.grad_done >= t - 1 and c.started == c.written:
        if grant_before_wait or t == 0 or peer.started >= t:
            c.started = t
            progress = True
    t = c.written + 1  # softmax end: the partner's grant received, tile written, copy issued
    if t <= c.started and (t == 0 or peer.started >= t):
        c.written = t
        progress = True
    if c.flushed < c.blocks and c.staged > c.flushed // c.nb:  # flush
        c.flushed += 1
        c.tiles_flushed = c.flushed // c.nb
        progress = True
    return progress


def simulate(ntiles, slots=4, grant_before_wait=True):
    a, b = Cta(0, ntiles, slots), Cta(1, ntiles, slots)
    progress = True
    while progress:
        progress = step(a, b, grant_before_wait) | step(b, a, grant_before_wait)
    return a.done() and b.done()


def test_schedule_covers_every_item_once():
    for rank in (0, 1):
        for nt in (1, 2, 5):
            ev = schedule(rank, nt)
            assert sorted(e for e in ev if e[1] == "S") == [(i, "S", j, 0) for i in range(nt) for j in range(14)]
            g = sorted(e for e in ev if e[1] == "G")
            assert g == [(i, "G", k, h) for i in range(nt) for k in range(nblocks(rank))
                         for h in range(1 if k < 5 else 2)]


@pytest.mark.parametrize("ntiles", [1, 2, 3, 8])
def test_pair_schedule_is_deadlock_free(ntiles):
    assert simulate(ntiles)


@pytest.mark.parametrize("inter", [0, 1, 2, 3, 4])
def test_every_group_placement_is_deadlock_free(inter):
    """Whole triples after any five consecutive blocks keep the ring live (the placement is a
    performance choice only)."""
    global INTER
    saved = INTER
    INTER = inter
    try:
        assert all(simulate(n) for n in (1, 2, 3, 8))
    finally:
        INTER = saved


def test_model_detects_a_deadlock():
    """Not vacuous: a CTA that waited for its partner's grant before sending its own would
    deadlock both, and a 2-slot ring cannot hold a key chunk across its S / dP items."""
    assert not simulate(3, grant_before_wait=False)
    assert not simulate(3, slots=2)


def test_pairs_of_items_deadlock_a_four_slot_ring():
    """The single-row kernel's interleave (two items after each of the last seven blocks) puts
    a two-chunk gradient block between a key chunk and its dO chunk: with four slots the held
    key chunk blocks the ring.  Whole triples do not."""
    def two_per_block(rank, ntiles):
        nb = nblocks(rank)
        ev = [(0, "S", j, 0) for j in range(14)]
        for i in range(ntiles):
            for k in range(nb):
                for h in range(1 if k < 5 else 2):
                    ev.append((i, "G", k, h))
                if i + 1 < ntiles and k >= nb - 7:
                    ev += [(i + 1, "S", 2 * (k - nb + 7) + q, 0) for q in range(2)]
        return ev
    global schedule
    saved = schedule
    schedule = two_per_block
    try:
        assert not simulate(3)
    finally:
        schedule = saved
    assert simulate(3)


# ---------------------------------------------------------------------------
# The merged schedule: the next tile's S / dP items share the own row's chunk
# ---------------------------------------------------------------------------
# Per tile after the five dQ~ blocks, for c = 0..4: the key-side block c (rank 0 dV c < 4,
# rank 1 dK~ c < 5; loads: own chunk, partner chunk) followed by the next tile's S item c
# (K_c', own q chunk) and dP item c (c < 4: K_c', own dO chunk).  When the next tile belongs
# to the same pair, the own chunk of the key-side block is also the S item's q chunk (rank 1)
# or the dP item's dO chunk (rank 0): it is loaded once and its slot is released after its
# second use.  Loads are FIFO in the ring; a slot is freed after the last MMA that reads it.

def merged_ops(rank, ntiles, same=True):
    """(loads, mmas): loads in issue order; mmas in issue order as (kind, tile, block, [load ids]).
    kind: 'S' (an S / dP item; 'S13' marks the tile's last), 'G' (first half of a gradient block,
    needs staging, and for block 0 the tile's P / dS), 'H' (second half), 'Gq' (a one-chunk dQ~ block)."""
    nkey = 5 if rank else 4
    loads, mmas = [], []

    def ld(tag):
        loads.append(tag)
        return len(loads) - 1

    def sdp_items(i, c, sq=None, so=None):
        k = ld(("K", i, c))
        q = sq if sq is not None else ld(("Q", i, c))
        mmas.append(("S", i, 2 * c, [k, q]))
        if c < 4:
            o = so if so is not None else ld(("O", i, c))
            mmas.append(("S", i, 2 * c + 1, [k, o]))
        if c == 4:
            mmas[-1] = ("S13", i, 2 * c, [k, q])

    for c in range(5):  # the first tile's S / dP, standalone
        sdp_items(0, c)
    for i in range(ntiles):
        nxt = i + 1 < ntiles
        for c in range(5):
            mmas.append(("Gq", i, c, [ld(("Kq", i, c))]))
        for c in range(5):
            own = None
            if c < nkey:
                own = ld(("own", i, c))
                par = ld(("par", i, c))
                mmas.append(("G", i, 5 + c, [own]))
                mmas.append(("H", i, 5 + c, [par]))
            if nxt:
                share = same and own is not None
                if rank == 1:
                    sdp_items(i + 1, c, sq=own if share else None)
                else:
                    sdp_items(i + 1, c, so=own if share and c < 4 else None)
    return loads, mmas


def simulate_merged(ntiles, slots=(4, 5), same=True):
    """Both CTAs' merged schedules against the ring, staging, softmax / exchange and flush rules.
    `slots`: ring slots of rank 0 and rank 1 (rank 1 stores its P straight into the partner's
    receive buffer, so its own P buffer serves as a fifth slot); an int gives both the same."""
    if isinstance(slots, int):
        slots = (slots, slots)
    class C:
        pass

    ctas = []
    for rank in (0, 1):
        c = C()
        c.rank = rank
        c.slots = slots[rank]
        c.loads, c.mmas = merged_ops(rank, ntiles, same)
        last_use = {}
        for mi, (_, _, _, ids) in enumerate(c.mmas):
            for l in ids:
                last_use[l] = mi
        c.release_at = last_use
        c.nb = 9 if rank == 0 else 10
        c.loaded = c.issued = c.flushed = c.blocks = 0
        c.freed = set()
        c.started = c.written = c.sdp_done = c.grad_done = -1
        ctas.append(c)

    def step(c, peer):
        progress = False
        if c.loaded < len(c.loads):  # producer: FIFO ring
            if c.loaded < c.slots or (c.loaded - c.slots) in c.freed:
                c.loaded += 1
                progress = True
        if c.issued < len(c.mmas):  # MMA
            kind, i, b, ids = c.mmas[c.issued]
            ready = all(l < c.loaded for l in ids)
            if kind in ("G", "Gq"):
                if b == 0 and c.written < i:
                    ready = False
                if c.blocks >= 2 and c.flushed < c.blocks - 1:
                    ready = False
            if kind == "H" and b == 5 and peer.written < i:
                ready = False
            if ready:
                if kind in ("G", "Gq"):
                    c.blocks += 1
                if kind in ("H", "Gq") and b == c.nb - 1:
                    c.grad_done = i
                if kind == "S13":
                    c.sdp_done = i
                c.freed.update(l for l, at in c.release_at.items() if at == c.issued)
                c.issued += 1
                progress = True
        t = c.started + 1
        if t < ntiles and c.sdp_done >= t and c.grad_done >= t - 1 and c.started == c.written:
            c.started = t
            progress = True
        t = c.written + 1
        if t <= c.started and (t == 0 or peer.started >= t):
            c.written = t
            progress = True
        if c.flushed < c.blocks:
            c.flushed += 1
            progress = True
        return progress

    a, b = ctas
    progress = True
    while progress:
        progress = step(a, b) | step(b, a)
    return all(c.loaded == len(c.loads) and c.issued == len(c.mmas) and c.written == ntiles - 1 for c in ctas)


@pytest.mark.parametrize("ntiles", [1, 2, 3, 8])
@pytest.mark.parametrize("same", [True, False])
@pytest.mark.parametrize("slots", [(4, 5), 4])
def test_merged_schedule_is_deadlock_free(ntiles, same, slots):
    assert simulate_merged(ntiles, slots=slots, same=same)


def test_merged_schedule_loads():
    """Per tile: rank 0 23 chunk loads (27 without sharing), rank 1 24 (29)."""
    for rank, shared, unshared in ((0, 23, 27), (1, 24, 29)):
        n2 = len(merged_ops(rank, 2, True)[0]) - len(merged_ops(rank, 1, True)[0])
        u2 = len(merged_ops(rank, 2, False)[0]) - len(merged_ops(rank, 1, False)[0])
        assert (n2, u2) == (shared, unshared)


def test_merged_model_detects_a_deadlock():
    assert not simulate_merged(3, slots=2)
    assert not simulate_merged(3, slots=(2, 5))
