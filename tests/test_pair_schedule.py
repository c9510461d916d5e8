"""Deadlock check of the paired-row backward's schedule (two CTAs of a cluster), on the CPU.

Each CTA has two rings of 32 KB operand slots, each with its own producer and MMA warp: the
gradient ring carries, per tile, the five key chunks of the dQ~ blocks and then each key-side
block's own-row and partner chunk (rank 0 dV 0-3, rank 1 dK~ 0-4); the S / dP ring carries each
tile's S items (K_c, q_c) and dP items (K_c, dO_c).  The CTAs are coupled through the exchanged
P / dS tile:
  * softmax of tile i starts when its S / dP items were issued and its own gradient MMAs of
    tile i - 1 completed; at its start it grants the partner the copy of tile i, then (i >= 1)
    waits for the partner's grant before writing; when the tile is written the copy is issued;
  * the S / dP MMA warp starts tile i's items once the softmax has read tile i - 1's S^T / dP^T;
  * the gradient MMA warp's first dQ~ block needs the tile's P / dS, the second half of the first
    key-side block the partner's copy; a gradient block needs a free staging buffer (two,
    released by the flush in order).
The model replays both CTAs against these dependencies and checks that every role finishes.
"""
import pytest

# ---------------------------------------------------------------------------------------------
# Two rings, two MMA warps: the gradient blocks (dQ~ key chunks, the key-side blocks' own and
# partner chunks) stream through one ring consumed by one MMA warp; the next tile's S / dP items
# (S item (K_c, Q_c), dP item (K_c, dO_c): the key chunk loaded for each item) through a second
# ring consumed by a second MMA warp, which starts a tile's items once the softmax has read the
# previous tile's S^T / dP^T.  Each ring has its own producer warp.
# ---------------------------------------------------------------------------------------------
def two_ring_ops(rank, ntiles, hold_k=False):
    """Per CTA: gradient ops [(kind, tile, block, n_chunks)], S ops [(tile, last, n_chunks)]: items
    of two chunks, or with hold_k (an S ring of 3+ slots keeps K_c from S item c to dP item c) one
    op per c of three chunks (c < 4) or two (c = 4); `last` marks the tile's last op."""
    nkey = 5 if rank else 4
    grad = []  # (kind, tile, block, chunks needed present, chunks released)
    for i in range(ntiles):
        if rank:  # own dQ~ 0-3, rank 0's dQ~ 3 (same key chunk, needs rank 0's dS), own dQ~ 4
            grad += [("Gq", i, c, 1, 1) for c in range(3)]
            grad += [("Gq", i, 3, 1, 0), ("Gm", i, 4, 1, 1), ("Gq", i, 5, 1, 1)]
        else:     # dQ~ 0, 1, 2, 4
            grad += [("Gq", i, c, 1, 1) for c in range(4)]
        nq = 6 if rank else 4
        for c in range(nkey):
            grad += [("G", i, nq + c, 1, 1), ("H", i, nq + c, 1, 1)]
    if hold_k:
        sdp = [(i, c == 4, 3 if c < 4 else 2) for i in range(ntiles) for c in range(5)]
    else:
        sdp = [(i, j == 8, 2) for i in range(ntiles) for j in range(9)]  # 5 S items + 4 dP items
    return grad, sdp


def simulate_two_rings(ntiles, gslots=(2, 3), sslots=(2, 2)):
    class C:
        pass

    ctas = []
    for rank in (0, 1):
        c = C()
        c.rank = rank
        c.gs, c.ss = gslots[rank], sslots[rank]
        c.grad, c.sdp = two_ring_ops(rank, ntiles, hold_k=c.ss >= 3)
        c.nb = 8 if rank == 0 else 11
        c.gl = c.gi = 0  # gradient chunks loaded / ops issued
        c.gused = 0      # gradient chunks released
        c.sl = c.si = 0  # S chunks loaded / S ops issued
        c.sused = 0      # S chunks released
        c.flushed = c.blocks = 0
        c.started = c.written = -1
        c.sdp_done = -1   # last tile whose S / dP items were all issued
        c.grad_done = -1  # last tile whose last key-side MMA was issued
        ctas.append(c)

    def step(c, peer):
        progress = False
        if c.gl < sum(op[4] for op in c.grad) and c.gl - c.gused < c.gs:  # gradient producer
            c.gl += 1
            progress = True
        if c.sl < sum(n for _, _, n in c.sdp) and c.sl - c.sused < c.ss:  # S producer
            c.sl += 1
            progress = True
        if c.gi < len(c.grad):  # gradient MMA warp
            kind, i, b, need, rel = c.grad[c.gi]
            ready = c.gl >= c.gused + need
            if kind in ("G", "Gq", "Gm"):
                if b == 0 and c.written < i:
                    ready = False
                if c.blocks >= 2 and c.flushed < c.blocks - 1:
                    ready = False
            nq = 6 if c.rank else 4
            if kind == "Gm" and peer.written < i:  # rank 0's dS of tile i
                ready = False
            if kind == "H" and b == nq and c.rank == 0 and peer.written < i:  # rank 1's P of tile i
                ready = False
            if ready:
                if kind in ("G", "Gq", "Gm"):
                    c.blocks += 1
                if kind == "H" and b == c.nb - 1:
                    c.grad_done = i
                c.gused += rel
                c.gi += 1
                progress = True
        if c.si < len(c.sdp):  # S MMA warp: tile i's items after the softmax read tile i - 1's
            i, last, n = c.sdp[c.si]
            if c.sl >= c.sused + n and (i == 0 or c.started >= i - 1):
                if last:
                    c.sdp_done = i
                c.sused += n
                c.si += 1
                progress = True
        t = c.started + 1  # softmax of tile t (grants the partner's copy)
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
    return all(c.gi == len(c.grad) and c.si == len(c.sdp) and c.written == ntiles - 1 for c in ctas)


@pytest.mark.parametrize("ntiles", [1, 2, 3, 8])
@pytest.mark.parametrize("gslots,sslots", [((2, 2), (2, 3)), ((2, 3), (2, 2)), ((1, 2), (3, 3)),
                                           ((1, 1), (3, 4)), ((1, 1), (2, 2))])
def test_two_ring_schedule_is_deadlock_free(ntiles, gslots, sslots):
    assert simulate_two_rings(ntiles, gslots, sslots)


def test_two_ring_model_detects_a_deadlock():
    """An S ring of one slot cannot hold an item's two chunks."""
    assert not simulate_two_rings(3, (2, 3), (1, 2))
