"""A randomised model of the prefill ring kernel's cross-CTA protocol (csrc/chunk_tc3.cuh), checked
on the CPU: two CTAs, each with a local role (chunk-local factors of every other chunk, written
into slot c % 3 of both CTAs) and a chain role (the serial state pass over every chunk), and the
three per-slot barriers:

  full[j]  completes when the producing CTA's local role has arrived (its own slot) or when the
           peer's remote arrive.expect_tx has been made and every copied byte has landed;
  free[j]  (count 2) in the CTA producing the slot's next chunk: both chains are done with it;
  land[j]  in the producing CTA: the other CTA has received the slot, so the copies out of it are
           done and the producer's chain may write U into it.

Every role takes its steps in the kernel's order, interleaved at random with the landing of the
asynchronous copies.  The model asserts that no slot is overwritten (by TMA or by copies) before
both chains released its previous chunk, that a chain reads a slot only when it holds its chunk,
that U is written only after the copies out of the slot landed, and that no schedule deadlocks.
"""
import random

import pytest

NSLOT = 3


class Barrier:
    """mbarrier with an arrival count and a transaction count; `done` counts completed phases."""

    def __init__(self, count):
        self.count, self.pending, self.tx, self.done = count, count, 0, 0

    def arrive(self, tx=0):
        self.tx += tx
        self.pending -= 1
        self._check()

    def complete_tx(self, n):
        self.tx -= n
        self._check()

    def _check(self):
        assert self.pending >= 0
        if self.pending == 0 and self.tx == 0:
            self.done += 1
            self.pending = self.count

    def passed(self, parity):  # try_wait.parity: the phase with this parity has completed
        return (self.done & 1) != parity


def run(nchunks, seed, skip_land_wait=False):
    rng = random.Random(seed)
    cta = [dict(full=[Barrier(1) for _ in range(NSLOT)], free=[Barrier(2) for _ in range(NSLOT)],
                land=[Barrier(1) for _ in range(NSLOT)]) for _ in range(2)]
    released = {}       # chunk -> ranks whose chain is done with it
    slot_chunk = {}     # (rank, slot) -> chunk whose data the slot holds
    landed = {}         # chunk -> every copy into the other CTA has landed
    inflight = []       # asynchronous copy completions not yet delivered

    def slot_free_for(c):  # both chains are done with chunk c - 3
        return c < NSLOT or released.get(c - NSLOT, set()) == {0, 1}

    def local(r):
        ph_free, c, peer = 0, r, r ^ 1
        if c < nchunks:
            assert slot_free_for(c), ("raw q/k loaded into a busy slot", c)
            slot_chunk[(r, c % NSLOT)] = c
        while c < nchunks:
            j = c % NSLOT
            yield None  # K1, m1
            # Qh, Ac, gamma_C start moving to the peer: remote expect_tx for both copy batches
            assert slot_free_for(c), ("copies into a busy peer slot", c)
            cta[peer]["full"][j].arrive(tx=2)
            slot_chunk[(peer, j)] = c
            inflight.append(lambda peer=peer, j=j: cta[peer]["full"][j].complete_tx(1))
            yield None  # inverse, m2
            issued = False
            if c + 2 < nchunks:  # raw q/k of own chunk c + 2, if its slot is already free
                jn = (c + 2) % NSLOT
                if c + 2 < NSLOT:
                    issued = True
                elif cta[r]["free"][jn].passed((ph_free >> jn) & 1):
                    ph_free ^= 1 << jn
                    issued = True
                if issued:
                    assert slot_free_for(c + 2), ("raw q/k loaded into a busy slot", c + 2)
                    slot_chunk[(r, jn)] = c + 2
            yield None  # E2, E1b
            # hand-off: the rest of the slot to the peer, local arrive on full
            def last(peer=peer, j=j, c=c):
                cta[peer]["full"][j].complete_tx(1)
                landed[c] = True
            inflight.append(last)
            cta[r]["full"][j].arrive()
            if c + 2 < nchunks and not issued:
                jn = (c + 2) % NSLOT
                while not cta[r]["free"][jn].passed((ph_free >> jn) & 1):
                    yield "wait"
                ph_free ^= 1 << jn
                assert slot_free_for(c + 2), ("raw q/k loaded into a busy slot", c + 2)
                slot_chunk[(r, jn)] = c + 2
            c += 2

    def chain(r):
        ph_full = ph_land = 0
        peer = r ^ 1
        for c in range(nchunks):
            j = c % NSLOT
            producer = (c & 1) == r
            while not cta[r]["full"][j].passed((ph_full >> j) & 1):
                yield "wait"
            ph_full ^= 1 << j
            assert slot_chunk.get((r, j)) == c, ("state pass reads the wrong chunk", r, c)
            if not producer:
                cta[peer]["land"][j].arrive()  # this CTA has received the slot
            yield None  # MMA group 1
            if producer:
                if not skip_land_wait:
                    while not cta[r]["land"][j].passed((ph_land >> j) & 1):
                        yield "wait"
                    ph_land ^= 1 << j
                assert landed.get(c), ("U written before the copies out of the slot landed", c)
            yield None  # E3, MMA group 2
            released.setdefault(c, set()).add(r)
            cta[(c + NSLOT) & 1]["free"][j].arrive()  # the CTA producing chunk c + 3
            yield None  # E4

    roles = [local(0), local(1), chain(0), chain(1)]
    alive, stall = list(range(4)), 0
    while alive or inflight:
        if inflight and (not alive or rng.random() < 0.3):
            inflight.pop(rng.randrange(len(inflight)))()
            stall = 0
            continue
        i = rng.choice(alive)
        try:
            if next(roles[i]) == "wait":
                stall += 1
                if stall > 10000 and not inflight:
                    raise RuntimeError("deadlock")
            else:
                stall = 0
        except StopIteration:
            alive.remove(i)
    assert released == {c: {0, 1} for c in range(nchunks)}


@pytest.mark.parametrize("nchunks", [1, 2, 3, 4, 5, 6, 7, 9, 17, 64])
def test_ring_protocol_random_schedules(nchunks):
    for seed in range(300):
        run(nchunks, seed)


def test_model_catches_a_missing_land_wait():
    """Without the producer's wait on land[j], some schedule writes U before the copies landed."""
    with pytest.raises(AssertionError, match="U written before"):
        for seed in range(300):
            run(9, seed, skip_land_wait=True)
