"""Deadlock check of the fused backward's cross-tile schedule, on the CPU.

The producer and MMA warps walk a CTA's tiles with one tile of lookahead: each tile's 14
gradient blocks (dQ~ 0-4, dK~ 0-4, dV 0-3, one chunk load each) with the next tile's 14
S / dP items (K0 Q0 O0 ... K3 Q3 O3 K4 Q4) interleaved two after each of the last seven
blocks.  This model replays that schedule against the kernel's dependencies and checks
that every role finishes:
  * ring: a load waits until the item `slots` earlier has been released; Q / O chunks are
    released by their S / dP MMA, a key chunk by its dP MMA (by S for the rope chunk), a
    gradient chunk by its block's MMA;
  * MMA: block 0 of a tile waits for that tile's softmax; block b waits until the flush
    has finished block b - 2 (two TMEM staging slots);
  * softmax of tile i waits for its S / dP (item 13 issued) and for tile i - 1's last
    gradient block (P / dS buffers);
  * flush: blocks in issue order, after the tile's row ids are staged; the producer stages
    tile i's row ids (when it starts tile i's S / dP items) only after the flush has
    finished tile i - 2 (two row-id buffers).
"""
import pytest

INTERLEAVE = 7   # first gradient block followed by next-tile S / dP items
PER_BLOCK = 2    # S / dP items after each of those blocks


def sdp_item(j):
    c = j // 3
    return j - 3 * c, c  # kind (0 key, 1 q, 2 dO), chunk


def schedule(ntiles):
    ev = [(0, "S", j) for j in range(14)]
    for i in range(ntiles):
        for k in range(14):
            ev.append((i, "G", k))
            if i + 1 < ntiles and k >= INTERLEAVE:
                ev += [(i + 1, "S", PER_BLOCK * (k - INTERLEAVE) + q) for q in range(PER_BLOCK)]
    return ev


def release_points(ev):
    """Event index after whose MMA each loaded item's slot is free."""
    rel = {}
    for idx, (i, typ, x) in enumerate(ev):
        if typ == "G":
            rel[idx] = idx
            continue
        kind, c = sdp_item(x)
        if kind != 0:
            rel[idx] = idx
        if kind == 2 or c == 4:  # releases the key chunk of this S / dP pair
            kidx = max(e for e in range(idx + 1) if ev[e] == (i, "S", 3 * c))
            rel[kidx] = idx
    return rel


def simulate(ntiles, slots):
    ev = schedule(ntiles)
    n = len(ev)
    rel = release_points(ev)
    loaded = issued = flushed = 0
    freed = set()
    staged = 0            # tiles whose row ids are staged
    softmax = -1          # last tile whose P / dS are written
    sdp_done = -1         # last tile whose S / dP item 13 was issued
    grad_done = -1        # last tile whose gradient block 13 was issued
    blocks = 0            # gradient blocks issued
    tiles_flushed = 0
    progress = True
    while progress:
        progress = False
        if loaded < n:  # producer
            i, typ, x = ev[loaded]
            ready = True
            if typ == "S" and x == 0 and staged <= i:
                if tiles_flushed < i - 1:
                    ready = False
                else:
                    staged = i + 1
            if ready and loaded >= slots and (loaded - slots) not in freed:
                ready = False
            if ready:
                loaded += 1
                progress = True
        if issued < loaded:  # MMA
            i, typ, x = ev[issued]
            ready = True
            if typ == "G" and ((x == 0 and softmax < i) or (blocks >= 2 and flushed < blocks - 1)):
                ready = False
            if ready:
                if typ == "G":
                    blocks += 1
                    grad_done = i if x == 13 else grad_done
                elif x == 13:
                    sdp_done = i
                freed.update(k for k, r in rel.items() if r == issued)
                issued += 1
                progress = True
        t = softmax + 1  # softmax
        if t < ntiles and sdp_done >= t and grad_done >= t - 1:
            softmax = t
            progress = True
        if flushed < blocks and staged > flushed // 14:  # flush
            flushed += 1
            tiles_flushed = flushed // 14
            progress = True
    return loaded == n and issued == n and flushed == 14 * ntiles and softmax == ntiles - 1


def test_schedule_covers_every_item_once():
    for nt in (1, 2, 5):
        ev = schedule(nt)
        assert sorted(e for e in ev if e[1] == "S") == [(i, "S", j) for i in range(nt) for j in range(14)]
        assert sorted(e for e in ev if e[1] == "G") == [(i, "G", k) for i in range(nt) for k in range(14)]


@pytest.mark.parametrize("slots", [5, 6])  # the ring sizes of N1 = 128 and N1 = 64
@pytest.mark.parametrize("ntiles", [1, 2, 3, 8])
def test_schedule_is_deadlock_free(slots, ntiles):
    assert simulate(ntiles, slots)


def test_model_detects_a_deadlock():
    """The model is not vacuous: a 2-slot ring cannot hold a key chunk across its Q and dO
    items plus the interleaved stream, and the model reports it."""
    assert not simulate(3, 2)
