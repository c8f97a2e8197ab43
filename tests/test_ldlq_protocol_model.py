"""A host-side model of the barrier protocol of the H-aware sequential
assignment in csrc/ldlq.cu (ldlq_kernel), run under random interleavings.

Roles, one step at a time, over the K / 64 blocks b of the CTA's rows:
- the producer (warp 9) waits for dempty[b & 1] in phase ((b >> 1) & 1) ^ 1
  and loads block b's diagonal tile of U; then for every earlier block c it
  waits for ring stage empty[s] and loads the tile U[c][b] with, for c <= b - 2,
  the errors of block c from the workspace -- before the chunk c = b - 2 it
  waits for ebar[b & 1] in phase ((b - 2) >> 1) & 1 (block b - 2 stored);
- the in-order warp (warp 8) waits for tready in phase (b - 1) & 1 (T_b
  summed, b > 0) and for dfull[b & 1], rounds block b reading T_b and the
  diagonal tile, writes its errors to shared memory (est) and the workspace,
  and arrives on eready, then on ebar[b & 1], then on dempty[b & 1];
- the eight product warps form T_b for b = 1 .. nb - 1: per chunk c < b they
  wait for full[s] (and for the last chunk c = b - 1 for eready in phase
  (b - 1) & 1, reading est instead of the stage's errors), release the stage
  on empty[s], then sum their partials between two barriers of the eight
  warps, write T_b and arrive on tready.

The workspace errors of block b are stored before the in-order warp arrives
on ebar[b & 1] (fence.proxy.async in the kernel), so a copy started after the
wait reads them.  The model checks that every read sees the data of its own
block (T_b, est, the diagonal tile, the stage's U tile and errors), that no
buffer is rewritten while read, and that nothing deadlocks -- and that one
shared ebar barrier for both parities of b, instead of two, can stall the
producer on a phase that has already gone by.
"""

import random

import pytest

STAGES, PRODUCT_WARPS = 3, 8


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.tx, self.phase = count, count, 0, 0

    def _advance(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, "more arrivals than the phase counts"
        self._advance()

    def arrive_expect_tx(self, n):
        self.tx += n
        self.arrive()

    def complete_tx(self, n):
        self.tx -= n
        assert self.tx >= 0
        self._advance()

    def done(self, parity):
        return (self.phase & 1) != parity


def run(nb, seed, two_ebar=True):
    rng = random.Random(seed)
    full = [Bar(1) for _ in range(STAGES)]
    empty = [Bar(PRODUCT_WARPS) for _ in range(STAGES)]
    dfull, dempty = [Bar(1) for _ in range(2)], [Bar(1) for _ in range(2)]
    tready, eready = Bar(PRODUCT_WARPS), Bar(1)
    ebar = [Bar(1), Bar(1)] if two_ebar else [Bar(1)] * 2

    stage = [None] * STAGES          # (b, c, errors-of-block or None) a stage holds
    stage_readers = [0] * STAGES
    diag = [None, None]              # block whose diagonal tile each buffer holds
    diag_reading = [False, False]
    est = [None]                     # block whose errors est holds
    est_readers = [0]
    tbuf = [None]                    # block b whose T_b tbuf holds
    tbuf_reading = [False]
    stored = set()                   # blocks whose errors the workspace holds
    landings = []
    sync = {"gen": 0, "count": 0}    # the product warps' named barrier

    def producer():
        seq = 0
        for b in range(nb):
            db = b & 1
            yield lambda db=db, b=b: dempty[db].done(((b >> 1) & 1) ^ 1)
            assert not diag_reading[db]
            dfull[db].arrive_expect_tx(1)

            def land_d(db=db, b=b):
                diag[db] = b
                dfull[db].complete_tx(1)
            landings.append(land_d)
            for c in range(b):
                s = seq % STAGES
                yield lambda s=s, seq=seq: empty[s].done(((seq // STAGES) & 1) ^ 1)
                with_e = c + 1 < b
                if with_e and c == b - 2:
                    if two_ebar:  # ebar[b & 1] completes one phase per block of that parity
                        yield lambda b=b: ebar[b & 1].done(((b - 2) >> 1) & 1)
                    else:         # one barrier, one phase per block
                        yield lambda b=b: ebar[0].done((b - 2) & 1)
                if with_e:
                    assert c in stored, ("errors of block", c, "copied before they were stored")
                assert stage_readers[s] == 0, "stage refilled while the product warps read it"
                full[s].arrive_expect_tx(1)

                def land(s=s, b=b, c=c, with_e=with_e):
                    stage[s] = (b, c, c if with_e else None)
                    full[s].complete_tx(1)
                landings.append(land)
                seq += 1

    def in_order():
        for b in range(nb):
            db = b & 1
            if b > 0:
                yield lambda b=b: tready.done((b - 1) & 1)
                assert tbuf[0] == b, ("rounding block", b, "with T of", tbuf[0])
            yield lambda db=db, b=b: dfull[db].done((b >> 1) & 1)
            assert diag[db] == b, ("rounding block", b, "with the diagonal tile of", diag[db])
            tbuf_reading[0] = True
            diag_reading[db] = True
            assert est_readers[0] == 0, "est rewritten while the product warps read it"
            yield None  # rounds the block
            est[0] = b
            stored.add(b)
            tbuf_reading[0] = False
            diag_reading[db] = False
            eready.arrive()
            ebar[db].arrive()
            dempty[db].arrive()

    def product(w):
        seq = 0
        for b in range(1, nb):
            for c in range(b):
                s = seq % STAGES
                yield lambda s=s, seq=seq: full[s].done((seq // STAGES) & 1)
                assert stage[s][:2] == (b, c), ("product read tile", stage[s], "expected", (b, c))
                if c + 1 == b:
                    yield lambda b=b: eready.done((b - 1) & 1)
                    assert est[0] == b - 1, ("product read est of", est[0], "expected", b - 1)
                    est_readers[0] += 1
                else:
                    assert stage[s][2] == c
                stage_readers[s] += 1
                yield None  # the FMAs over the chunk
                stage_readers[s] -= 1
                if c + 1 == b:
                    est_readers[0] -= 1
                empty[s].arrive()
                seq += 1
            for _ in range(2):  # partials, then T_b: between two barriers of the eight warps
                gen = sync["gen"]
                sync["count"] += 1
                if sync["count"] == PRODUCT_WARPS:
                    sync["count"], sync["gen"] = 0, gen + 1
                yield lambda gen=gen: sync["gen"] > gen
                if _ == 0 and w == 0:
                    assert not tbuf_reading[0], "T rewritten while the in-order warp reads it"
                    tbuf[0] = b
            tready.arrive()

    actors = [producer(), in_order()] + [product(w) for w in range(PRODUCT_WARPS)]
    waits = [None] * len(actors)
    alive = list(range(len(actors)))
    while alive or landings:
        ready = [("step", i) for i in alive if waits[i] is None or waits[i]()]
        ready += [("land", j) for j in range(len(landings))]
        assert ready, f"deadlock: nb = {nb}"
        kind, i = rng.choice(ready)
        if kind == "land":
            landings.pop(i)()
        else:
            try:
                waits[i] = next(actors[i])
            except StopIteration:
                alive.remove(i)
    assert stored == set(range(nb))


@pytest.mark.parametrize("nb", [1, 2, 3, 4, 5, 8, 13])
def test_protocol_reads_its_own_blocks_without_deadlock(nb):
    for seed in range(40):
        run(nb, seed)


def test_one_ebar_for_both_parities_can_stall_the_producer():
    """With a single barrier (one phase per block, the wait for block b - 2 in
    parity (b - 2) & 1) the in-order warp can finish block b - 1 before the
    producer's wait: the barrier is then a phase further on, the wait's parity
    names a phase still to come (block b), and block b needs the very stages
    the producer holds back -- a deadlock on some schedules."""
    failures = 0
    for seed in range(200):
        try:
            run(8, seed, two_ebar=False)
        except AssertionError:
            failures += 1
    assert failures > 0
