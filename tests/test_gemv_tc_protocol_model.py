"""A host-side model of the barrier protocol of the tcgen05 decode-GEMV in
csrc/gemv_tc.cu (gemv_tc_kernel: large groups at 17..32 tokens), run under
random interleavings.

Roles, one step at a time (counters as in the kernel: g = the CTA's k-block
count, c = g / 4 its code chunk, `local` its tile count):
- the code producer waits for cempty[c % 4] in phase ((c / 4) & 1) ^ 1, arms
  cfull[c % 4] with the chunk's bytes and starts the copy;
- the X'' producer waits for aempty[g % 6] in phase ((g / 6) & 1) ^ 1, arms
  xfull[g % 6] and starts the copy;
- decoder warp (q, slot) takes the k-blocks with g % 4 == slot: it waits for
  cfull and aempty, writes its row quarter q of A slot g % 6, then arrives on
  cempty (16 arrivals per chunk) and afull (4 per slot);
- the MMA issuer waits for tempty[local & 1], then per k-block for afull and
  xfull, issues, and commits aempty; after the tile's last k-block it commits
  tfull;
- the four epilogue warps wait for tfull[local & 1], read D and arrive on
  tempty.

Copies land asynchronously in any order (complete_tx); commits arrive
asynchronously in issue order.  The barriers follow mbarrier phase semantics:
an arrival count and a transaction count per phase, and a parity wait that
passes once the phase of that parity has completed.  The model checks that
every k-block the MMA consumes holds that k-block's codes in all four row
quarters and its X'' tile, that no slot or accumulator is rewritten while in
use, that every tile's accumulator the epilogue reads is that tile's and
complete, and that nothing deadlocks.
"""

import random

import pytest

C_STAGES, A_STAGES, SUB, EPI = 4, 6, 4, 4


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


def run(tiles, seed, cempty_count=4 * SUB, tempty_count=EPI, decoder_waits_slot=True,
        mma_waits_x=True):
    """tiles: the number of code chunks (K / 512, rounded up) of each tile the
    CTA takes, in order."""
    rng = random.Random(seed)
    cfull = [Bar(1) for _ in range(C_STAGES)]
    cempty = [Bar(cempty_count) for _ in range(C_STAGES)]
    xfull = [Bar(1) for _ in range(A_STAGES)]
    afull = [Bar(4) for _ in range(A_STAGES)]
    aempty = [Bar(1) for _ in range(A_STAGES)]
    tfull = [Bar(1) for _ in range(2)]
    tempty = [Bar(tempty_count) for _ in range(2)]
    code = [None] * C_STAGES      # chunk held by each code stage
    xpp = [None] * A_STAGES       # k-block held by each X'' stage
    aslot = [[None] * 4 for _ in range(A_STAGES)]  # k-block per row quarter of each A slot
    in_use = [None] * A_STAGES    # k-block the MMAs still read from slot a
    dbuf = [None] * 2             # (tile, complete) held by each accumulator
    reads = [0] * 2               # epilogue warps that read the accumulator's tile
    landings, commits, consumed = [], [], []
    nkb = SUB * sum(tiles)

    def code_producer():
        for c in range(sum(tiles)):
            s = c % C_STAGES
            yield lambda s=s, c=c: cempty[s].done(((c // C_STAGES) & 1) ^ 1)
            cfull[s].arrive_expect_tx(1)

            def land(s=s, c=c):
                code[s] = c
                cfull[s].complete_tx(1)
            landings.append(land)

    def x_producer():
        for g in range(nkb):
            a = g % A_STAGES
            yield lambda a=a, g=g: aempty[a].done(((g // A_STAGES) & 1) ^ 1)
            assert in_use[a] is None, "X'' slot refilled while the MMAs read it"
            xfull[a].arrive_expect_tx(1)

            def land(a=a, g=g):
                xpp[a] = g
                xfull[a].complete_tx(1)
            landings.append(land)

    def decoder(q, slot):
        for g in range(slot, nkb, SUB):
            c = g // SUB
            s, a = c % C_STAGES, g % A_STAGES
            yield lambda s=s, c=c: cfull[s].done((c // C_STAGES) & 1)
            if decoder_waits_slot:
                yield lambda a=a, g=g: aempty[a].done(((g // A_STAGES) & 1) ^ 1)
            assert code[s] == c, ("decoder read chunk", code[s], "expected", c)
            assert in_use[a] is None, "A slot rewritten while the MMAs read it"
            aslot[a][q] = g
            cempty[s].arrive()
            afull[a].arrive()

    def mma():
        g = 0
        for local, nch in enumerate(tiles):
            buf = local & 1
            yield lambda buf=buf, local=local: tempty[buf].done(((local >> 1) & 1) ^ 1)
            if local >= 2:
                assert reads[buf] == EPI, "accumulator rewritten before the epilogue read it"
            dbuf[buf], reads[buf] = (local, False), 0
            for _ in range(SUB * nch):
                a, par = g % A_STAGES, (g // A_STAGES) & 1
                if mma_waits_x:
                    yield lambda a=a, par=par: afull[a].done(par) and xfull[a].done(par)
                else:
                    yield lambda a=a, par=par: afull[a].done(par)
                assert aslot[a] == [g] * 4 and xpp[a] == g, (g, aslot[a], xpp[a])
                in_use[a] = g
                consumed.append(g)

                def release(a=a):
                    in_use[a] = None
                    aempty[a].arrive()
                commits.append(release)
                g += 1

            def finish(buf=buf, local=local):
                dbuf[buf] = (local, True)
                tfull[buf].arrive()
            commits.append(finish)

    def epilogue():
        for local in range(len(tiles)):
            buf = local & 1
            yield lambda buf=buf, local=local: tfull[buf].done((local >> 1) & 1)
            assert dbuf[buf] == (local, True), ("epilogue read", dbuf[buf], "expected", local)
            reads[buf] += 1
            tempty[buf].arrive()

    actors = [code_producer(), x_producer(), mma()]
    actors += [decoder(q, s) for q in range(4) for s in range(SUB)]
    actors += [epilogue() for _ in range(EPI)]
    waits = [None] * len(actors)
    alive = list(range(len(actors)))
    while alive or landings or commits:
        ready = [("step", i) for i in alive if waits[i] is None or waits[i]()]
        ready += [("land", j) for j in range(len(landings))]
        ready += [("commit", 0)] if commits else []
        assert ready, f"deadlock: tiles {tiles}, {len(consumed)} k-blocks consumed"
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
    assert consumed == list(range(nkb))


def _cases(n):
    rng = random.Random(n)
    for seed in range(n):
        yield [rng.choice([1, 2, 3, 8, 9, 22]) for _ in range(rng.randint(1, 5))], seed


def test_protocol_consumes_every_k_block_in_order_without_deadlock():
    for tiles, seed in _cases(150):
        run(tiles, seed)


@pytest.mark.parametrize("mutation", [
    dict(decoder_waits_slot=False),   # a decoder that writes a slot before the MMAs let it go
    dict(mma_waits_x=False),          # an MMA that does not wait for X'' to land
    dict(cempty_count=4),             # a code stage released after one k-block's decoders
    dict(tempty_count=1),             # an accumulator released after one epilogue warp
])
def test_the_model_catches_a_broken_protocol(mutation):
    caught = False
    for tiles, seed in _cases(150):
        try:
            run(tiles, seed, **mutation)
        except AssertionError:
            caught = True
            break
    assert caught
