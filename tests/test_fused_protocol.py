"""CPU model of the fused append-read kernel's hand-over protocol (no GPU).

The kernel (append_read_fused_kernel in deferred_read.cu) has NP prep warps
and ND decode warps per block, synchronised by mbarriers in shared memory:
full[s] (the prep warp's 32 lanes arrive once its head's x_0 and w are in
slot s), free[s] (one arrival per decode unit of that head) and one ring
barrier per decode buffer (completed by the bulk copy's bytes). A wait names
the phase it needs by parity only, so an index or parity slip would either
block (the kernel's bounded wait then gives up) or, worse, let a warp read a
slot or buffer that holds another head's data.

This model runs the kernel's loops with the same index and parity formulas
as generators, one per warp, interleaved in random orders, with the hardware
rule for a parity wait (it passes once the barrier's completed-phase count
has the other parity). Every read must find the head or unit it expects,
every wait that passes must be for the phase it meant (never two phases
late), and every warp must finish: no order of the warps may deadlock.
"""
import random

import pytest


class Barrier:
    def __init__(self, count):
        self.count, self.pending, self.done = count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0
        if self.pending == 0:
            self.done += 1
            self.pending = self.count

    def passes(self, parity):
        return (self.done & 1) != parity


def run_block(nh, NP, ND, NBUF, UPH, seed):
    NSLOT = 2 * NP
    full = [Barrier(32) for _ in range(NSLOT)]
    free = [Barrier(UPH) for _ in range(NSLOT)]
    ring = [[Barrier(1) for _ in range(NBUF)] for _ in range(ND)]
    slot = [None] * NSLOT
    buf = [[None] * NBUF for _ in range(ND)]
    pending_copies = []  # (d, b, unit): a bulk copy in flight
    decoded = []

    def wait(bar, parity, expect_done):
        while not bar.passes(parity):
            yield
        # the phase it meant, not one two phases later with the same parity
        assert bar.done == expect_done, (bar.done, expect_done)

    def prep(p):
        for i in range(p, nh, NP):
            s = i % NSLOT
            if i >= NSLOT:
                yield from wait(free[s], (i // NSLOT - 1) & 1, i // NSLOT)
            yield
            slot[s] = i
            for _ in range(32):
                full[s].arrive()
            yield

    def decode(d):
        nf = nh * UPH

        def issue(f, b):
            pending_copies.append((d, b, f))

        issued = 0
        for b in range(NBUF):
            if d + b * ND < nf:
                issue(d + b * ND, b)
                issued += 1
        t = 0
        while True:
            f = d + t * ND
            if f >= nf:
                break
            b, i, s = t % NBUF, f // UPH, (f // UPH) % NSLOT
            yield from wait(ring[d][b], (t // NBUF) & 1, t // NBUF + 1)
            yield from wait(full[s], (i // NSLOT) & 1, i // NSLOT + 1)
            assert buf[d][b] == f, (buf[d][b], f)
            assert slot[s] == i, (slot[s], i)
            decoded.append(f)
            free[s].arrive()
            if f + NBUF * ND < nf:
                issue(f + NBUF * ND, b)
                issued += 1
            t += 1
            yield
        assert issued == t

    rng = random.Random(seed)
    warps = [prep(p) for p in range(NP)] + [decode(d) for d in range(ND)]
    live = list(range(len(warps)))
    steps = 0
    while live or pending_copies:
        steps += 1
        assert steps < 10_000_000, "no progress"
        if pending_copies and (not live or rng.random() < 0.3):
            k = rng.randrange(len(pending_copies))
            d, b, f = pending_copies.pop(k)
            buf[d][b] = f
            ring[d][b].arrive()
            continue
        if not live:
            continue
        w = rng.choice(live)
        try:
            next(warps[w])
        except StopIteration:
            live.remove(w)
    assert sorted(decoded) == list(range(nh * UPH))


# (heads of the block, NP, ND, NBUF, units per head): the shapes the layouts give
SHAPES = [(56, 11, 8, 3, 16), (55, 11, 8, 3, 16), (1, 11, 8, 3, 16), (13, 12, 8, 3, 4), (222, 8, 8, 3, 32),
          (23, 6, 8, 3, 16), (3, 8, 8, 3, 16), (100, 12, 8, 3, 8)]


@pytest.mark.parametrize("nh,NP,ND,NBUF,UPH", SHAPES)
def test_protocol_hands_over_every_head_in_any_order(nh, NP, ND, NBUF, UPH):
    for seed in range(4):
        run_block(nh, NP, ND, NBUF, UPH, seed)
