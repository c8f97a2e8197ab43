"""A host-side model of the barrier protocol of the single-CTA tcgen05 GEMM in
csrc/tc_gemm.cu (tc_gemm_kernel: the algebraic forward, dX and the Gram GEMM
of the full-H refit), run under random interleavings.

Roles, one step at a time, over the CTA's tiles and their k-blocks (one ring
of STAGES stages; each role walks it with its own stage index and phase bit):
- the producer waits for empty[s] in phase ph ^ 1, arms full[s] with the
  stage's bytes and starts the copies of A and of the packed codes;
- each of the DW decoder warps waits for full[s] in phase ph, decodes its rows
  of the codes into the stage's B tile and arrives on decd[s] (DW arrivals);
- the MMA issuer waits for tempty[local & 1], then per k-block for decd[s]
  (full[s] when the kind has no decoders), issues, and commits empty[s]; after
  the tile's last k-block it commits tfull;
- the four epilogue warps wait for tfull[local & 1], read D and arrive on
  tempty.

The decoders never wait for empty[s]: they are kept off a stage the MMAs still
read only because full[s] is re-armed after the MMAs' commit to empty[s].  The
model checks that property with the rest: every k-block the MMA consumes holds
that k-block's A, codes and decoded B; no copy or decoder overwrites a stage in
use; every accumulator the epilogue reads is that tile's, complete; nothing
deadlocks.  Copies land in any order, commits arrive in issue order.
"""

import random

import pytest

STAGES, EPI = 4, 4


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

    def done(self, parity):  # try_wait.parity: the phase with this parity has completed
        return (self.phase & 1) != parity


def run(ntiles, kblocks, DW, seed, producer_waits_empty=True, mma_waits_decoded=True,
        tempty_count=EPI, decd_count=None):
    rng = random.Random(seed)
    full = [Bar(1) for _ in range(STAGES)]
    decd = [Bar(decd_count or max(DW, 1)) for _ in range(STAGES)]
    empty = [Bar(1) for _ in range(STAGES)]
    tfull = [Bar(1) for _ in range(2)]
    tempty = [Bar(tempty_count) for _ in range(2)]
    stage_in = [None] * STAGES               # k-block whose A and codes a stage holds
    stage_b = [[None] * DW for _ in range(STAGES)]  # k-block each decoder's part of B holds
    in_use = [None] * STAGES                 # k-block the MMAs still read from the stage
    dbuf, reads = [None] * 2, [0] * 2
    landings, commits, consumed = [], [], []
    total = ntiles * kblocks

    def producer():
        for n in range(total):
            s, ph = n % STAGES, (n // STAGES) & 1
            if producer_waits_empty:
                yield lambda s=s, ph=ph: empty[s].done(ph ^ 1)
            full[s].arrive_expect_tx(1)

            def land(s=s, n=n):
                assert in_use[s] is None, "a copy overwrites a stage the MMAs still read"
                stage_in[s] = n
                full[s].complete_tx(1)
            landings.append(land)

    def decoder(w):
        for n in range(total):
            s, ph = n % STAGES, (n // STAGES) & 1
            yield lambda s=s, ph=ph: full[s].done(ph)
            assert stage_in[s] == n, ("decoder read the codes of", stage_in[s], "expected", n)
            assert in_use[s] is None, "a decoder overwrites B while the MMAs read it"
            stage_b[s][w] = n
            decd[s].arrive()

    def mma():
        n = 0
        for local in range(ntiles):
            buf = local & 1
            yield lambda buf=buf, local=local: tempty[buf].done(((local >> 1) & 1) ^ 1)
            if local >= 2:
                assert reads[buf] == EPI, "accumulator rewritten before the epilogue read it"
            dbuf[buf], reads[buf] = (local, False), 0
            for _ in range(kblocks):
                s, ph = n % STAGES, (n // STAGES) & 1
                ready = decd if (DW > 0 and mma_waits_decoded) else full
                yield lambda s=s, ph=ph, ready=ready: ready[s].done(ph)
                assert stage_in[s] == n, ("MMA read A of", stage_in[s], "expected", n)
                assert all(b == n for b in stage_b[s]), ("MMA read B of", stage_b[s], "expected", n)
                in_use[s] = n
                consumed.append(n)

                def release(s=s):
                    in_use[s] = None
                    empty[s].arrive()
                commits.append(release)
                n += 1

            def finish(buf=buf, local=local):
                dbuf[buf] = (local, True)
                tfull[buf].arrive()
            commits.append(finish)

    def epilogue():
        for local in range(ntiles):
            buf = local & 1
            yield lambda buf=buf, local=local: tfull[buf].done((local >> 1) & 1)
            assert dbuf[buf] == (local, True), ("epilogue read", dbuf[buf], "expected", local)
            reads[buf] += 1
            tempty[buf].arrive()

    actors = [producer(), mma()] + [decoder(w) for w in range(DW)] + [epilogue() for _ in range(EPI)]
    waits = [None] * len(actors)
    alive = list(range(len(actors)))
    while alive or landings or commits:
        ready = [("step", i) for i in alive if waits[i] is None or waits[i]()]
        ready += [("land", j) for j in range(len(landings))]
        ready += [("commit", 0)] if commits else []
        assert ready, f"deadlock: {ntiles} tiles x {kblocks} k-blocks, DW={DW}"
        kind, i = rng.choice(ready)
        if kind == "land":
            landings.pop(i)()
        elif kind == "commit":
            commits.pop(0)()
        else:
            try:
                waits[i] = next(actors[i])
            except StopIteration:
                alive.remove(i)
    assert consumed == list(range(total))


def _cases(n):
    rng = random.Random(7 * n)
    for seed in range(n):
        yield rng.randint(1, 5), rng.choice([1, 2, 3, 4, 5, 9, 64]), seed


@pytest.mark.parametrize("DW", [0, 4, 8])
def test_protocol_consumes_every_k_block_in_order_without_deadlock(DW):
    for ntiles, kblocks, seed in _cases(120):
        run(ntiles, kblocks, DW, seed)


@pytest.mark.parametrize("mutation", [
    dict(producer_waits_empty=False),  # copies that do not wait for the MMAs to release the stage
    dict(mma_waits_decoded=False),     # an MMA that takes the stage when the copies land
    dict(tempty_count=1),              # an accumulator released after one epilogue warp
    dict(decd_count=2),                # a stage counted as decoded after two of its decoders
])
def test_the_model_catches_a_broken_protocol(mutation):
    caught = False
    for ntiles, kblocks, seed in _cases(120):
        try:
            run(ntiles, kblocks, 4, seed, **mutation)
        except AssertionError:
            caught = True
            break
    assert caught
