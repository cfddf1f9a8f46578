"""A randomised model of the four-CTA prefill kernel's cross-CTA protocol (csrc/chunk_tc4.cuh),
checked on the CPU: four CTAs, each with a local role (the factors of chunks c with c % 4 == r,
built in a private working area and handed over through a per-producer staging entry in global
memory) and a chain role (the serial state pass over every chunk, with two factor slots filled
by bulk loads from the staging entries), and the barriers:

  ready[r]  (in every CTA, count 1) producer r's staging entry holds its next chunk;
  gfree     (in producer r, count 4) every chain has finished loading r's previous chunk;
  full[j]   (per chain, count 1 + bytes) slot j holds its chunk.

Every role takes its steps in the kernel's order, interleaved at random with the completion of
the asynchronous bulk loads.  The model asserts that a staging entry is not overwritten while a
load from it is in flight or still to come, that a slot is not refilled before its chain is done
with the chunk in it, that a chain reads a slot only when it holds its chunk, and that no schedule
deadlocks.
"""
import random

import pytest

NCTA, NSLOT = 4, 2


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


def run(nchunks, seed, skip_gfree_wait=False, eager_refill=False):
    rng = random.Random(seed)
    ready = [[Barrier(1) for _ in range(NCTA)] for _ in range(NCTA)]  # ready[cta][producer]
    gfree = [Barrier(NCTA) for _ in range(NCTA)]
    full = [[Barrier(1) for _ in range(NSLOT)] for _ in range(NCTA)]
    staging = [None] * NCTA            # producer -> chunk its entry holds
    slot = [[None] * NSLOT for _ in range(NCTA)]
    done_with = [-1] * NCTA            # chain -> last chunk whose output MMAs it has waited for
    inflight = []                      # bulk-load completions not yet delivered
    consumed = {}                      # chunk -> chains whose load of it has completed

    def local(r):
        ph_gfree = 0
        for c in range(r, nchunks, NCTA):
            yield None  # raw q/k, K1, m1, E1a, inverse, m2, E2/E1b in the working area
            if c >= NCTA and not skip_gfree_wait:
                while not gfree[r].passed(ph_gfree & 1):
                    yield "wait"
                ph_gfree ^= 1
            # bulk store of the block, waited for by the issuing thread, then the release arrives
            assert staging[r] is None or consumed.get(staging[r], set()) == set(range(NCTA)), (
                "staging entry overwritten before every chain loaded it", r, c)
            staging[r] = c
            for q in range(NCTA):
                ready[q][r].arrive()

    def chain(q):
        ph_full = ph_ready = 0
        n_loaded = 0

        def issue(x):  # bulk load of chunk x's block into slot x % 2
            nonlocal ph_ready, n_loaded
            r, j = x % NCTA, x % NSLOT
            assert done_with[q] >= x - NSLOT, ("slot refilled before its chunk was done", q, x)
            assert staging[r] == x, ("load from a staging entry holding another chunk", q, x, staging[r])
            ph_ready ^= 1 << r
            full[q][j].arrive(tx=1)

            def land(r=r, j=j, x=x):
                assert staging[r] == x, ("staging entry overwritten while a load from it was in flight", q, x)
                slot[q][j] = x
                consumed.setdefault(x, set()).add(q)
                full[q][j].complete_tx(1)
            inflight.append(land)
            n_loaded += 1

        def pump(last):
            while n_loaded <= last and n_loaded < nchunks:
                r = n_loaded % NCTA
                if not ready[q][r].passed((ph_ready >> r) & 1):
                    break
                issue(n_loaded)

        pump(NSLOT - 1)
        for c in range(nchunks + 1):
            run_c = c < nchunks
            if run_c:
                j = c % NSLOT
                if n_loaded == c:
                    r = c % NCTA
                    while not ready[q][r].passed((ph_ready >> r) & 1):
                        yield "wait"
                    issue(c)
                while not full[q][j].passed((ph_full >> j) & 1):
                    yield "wait"
                ph_full ^= 1 << j
                assert slot[q][j] == c, ("state pass reads the wrong chunk", q, c)
                gfree[c % NCTA].arrive()
                yield None  # MMA group 1 issued
            if c > 0:
                done_with[q] = c - 1  # the previous chunk's output MMAs waited for
                pump(c + 1 + (1 if eager_refill else 0))
            if not run_c:
                break
            yield None  # E3, MMA group 2
            pump(c + 1)
            yield None  # write vectors, U0 of the next chunk, E4

    roles = [local(r) for r in range(NCTA)] + [chain(q) for q in range(NCTA)]
    alive, stall = list(range(len(roles))), 0
    while alive or inflight:
        if inflight and (not alive or rng.random() < 0.3):
            inflight.pop(rng.randrange(len(inflight)))()
            stall = 0
            continue
        i = rng.choice(alive)
        try:
            if next(roles[i]) == "wait":
                stall += 1
                if stall > 20000 and not inflight:
                    raise RuntimeError("deadlock")
            else:
                stall = 0
        except StopIteration:
            alive.remove(i)
    assert consumed == {c: set(range(NCTA)) for c in range(nchunks)}


@pytest.mark.parametrize("nchunks", [1, 2, 3, 4, 5, 7, 8, 9, 17, 64])
def test_quad_protocol_random_schedules(nchunks):
    for seed in range(200):
        run(nchunks, seed)


def test_model_catches_a_missing_gfree_wait():
    """Without the producer's wait on gfree, some schedule overwrites a staging entry too early."""
    with pytest.raises(AssertionError, match="staging entry overwritten"):
        for seed in range(200):
            run(17, seed, skip_gfree_wait=True)


def test_model_catches_an_early_slot_refill():
    """Requesting chunk c+2 while chunk c's output MMAs may still read its slot is caught."""
    with pytest.raises(AssertionError, match="slot refilled before"):
        for seed in range(200):
            run(17, seed, eager_refill=True)
