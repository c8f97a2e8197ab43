"""A host-side model of the whole barrier protocol of the CTA-pair tcgen05 GEMM
in csrc/tc_gemm.cu (tc2_gemm_kernel: the decode-form forward and dW), run
under random interleavings.  tests/test_pair_handover_model.py covers the
grouped handover alone; this model adds the copies, the commits and the
accumulator's release across the pair.

Roles, one step at a time (ring of S stages, each role walks it with its own
stage index and phase bit; `it` counts the pair's k-blocks over its tiles):
- each CTA's producer waits for its own empty[s]; the even CTA arms fullA[s]
  with both CTAs' operand bytes (the pair's A and, without codes, B copies
  complete on the even CTA's barrier), each CTA arms its own fullC[s] with its
  codes and starts its copies;
- each CTA's decoder groups (group g takes the k-blocks with it % groups == g)
  wait for their CTA's fullC[s], decode that CTA's half of B and arrive on its
  decd[s] (one arrival per warp of the group);
- the odd CTA's forwarder waits for its decd[s] and, after the last k-block of
  each group of G (or the pair's very last k-block), arrives once on the even
  CTA's decd_peer[(it / G) % S];
- the even CTA's MMA issuer waits for tempty[local & 1] (both CTAs' epilogue
  warps), then per k-block for fullA[s], its own decd[s] and, at a group's
  first k-block, decd_peer[q % S] in phase (q / S) & 1; it issues and commits
  empty[s] to both CTAs (multicast), and after the tile tfull[buf] to both;
- the four epilogue warps of each CTA wait for their CTA's tfull, read its
  half of the accumulator and arrive on the even CTA's tempty.

Copies land in any order; commits arrive in issue order.  The model checks
that the MMA consumes every k-block in order with both CTAs' operands and both
B halves of that k-block, that no copy or decoder overwrites a stage the MMAs
still read, that each epilogue reads its tile's complete accumulator, and that
nothing deadlocks.
"""

import random

import pytest

S, G, EPI = 6, 3, 4


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
        # the transaction count may go below zero for a moment: the odd CTA's
        # copy can land on the even CTA's barrier before the even CTA's own
        # arrival announces the bytes; the phase still needs that arrival
        self.tx -= n
        self._advance()

    def done(self, parity):
        return (self.phase & 1) != parity


def run(ntiles, kblocks, groups, group_warps, codes, seed, multicast_empty=True,
        tempty_count=2 * EPI, mma_waits_peer=True, forward_at_first=False):
    rng = random.Random(seed)
    total = ntiles * kblocks
    fullA = [Bar(1) for _ in range(S)]                       # even CTA only
    fullC = [[Bar(1) for _ in range(S)] for _ in range(2)]
    decd = [[Bar(group_warps if codes else 1) for _ in range(S)] for _ in range(2)]
    empty = [[Bar(1) for _ in range(S)] for _ in range(2)]
    peer = [Bar(1) for _ in range(S)]
    tfull = [[Bar(1) for _ in range(2)] for _ in range(2)]
    tempty = [Bar(tempty_count) for _ in range(2)]
    opnd = [[None] * S for _ in range(2)]    # k-block whose operands each CTA's stage holds
    code = [[None] * S for _ in range(2)]    # k-block whose codes it holds
    bhalf = [[[None] * group_warps for _ in range(S)] for _ in range(2)]  # decoded B half
    in_use = [None] * S                      # k-block the MMAs still read from stage s
    dbuf = [[None, None] for _ in range(2)]  # per CTA and buffer: (tile, complete)
    reads = [[0, 0] for _ in range(2)]
    landings, commits, consumed = [], [], []

    def producer(c):
        for it in range(total):
            s, ph = it % S, (it // S) & 1
            yield lambda s=s, ph=ph: empty[c][s].done(ph ^ 1)
            assert in_use[s] is None, "stage refilled while the MMAs read it"
            if c == 0:
                fullA[s].arrive_expect_tx(2)
            if codes:
                fullC[c][s].arrive_expect_tx(1)

            def land_op(s=s, it=it):
                assert fullA[s].phase == it // S, "a copy landed in another phase of fullA"
                opnd[c][s] = it
                fullA[s].complete_tx(1)
            landings.append(land_op)
            if codes:
                def land_code(s=s, it=it):
                    assert fullC[c][s].phase == it // S, "a copy landed in another phase of fullC"
                    code[c][s] = it
                    fullC[c][s].complete_tx(1)
                landings.append(land_code)

    def decoder(c, grp, w):
        for it in range(total):
            if it % groups != grp:
                continue
            s, ph = it % S, (it // S) & 1
            yield lambda s=s, ph=ph: fullC[c][s].done(ph)
            assert code[c][s] == it, ("decoder read codes of", code[c][s], "expected", it)
            assert in_use[s] is None, "B half rewritten while the MMAs read it"
            bhalf[c][s][w] = it
            decd[c][s].arrive()

    def forwarder():
        for it in range(total):
            s, ph = it % S, (it // S) & 1
            yield lambda s=s, ph=ph: decd[1][s].done(ph)
            at = 0 if forward_at_first else G - 1
            if it % G == at or (not forward_at_first and it == total - 1):
                peer[(it // G) % S].arrive()

    def mma():
        it = 0
        for local in range(ntiles):
            buf = local & 1
            yield lambda buf=buf, local=local: tempty[buf].done(((local >> 1) & 1) ^ 1)
            if local >= 2:
                assert reads[0][buf] == EPI and reads[1][buf] == EPI, "accumulator reused early"
            for c in range(2):
                dbuf[c][buf], reads[c][buf] = (local, False), 0
            for _ in range(kblocks):
                s, ph = it % S, (it // S) & 1
                yield lambda s=s, ph=ph: fullA[s].done(ph)
                if codes:
                    yield lambda s=s, ph=ph: decd[0][s].done(ph)
                    if it % G == 0 and mma_waits_peer:
                        q = it // G
                        yield lambda q=q: peer[q % S].done((q // S) & 1)
                assert opnd[0][s] == it and opnd[1][s] == it, ("operands", opnd[0][s], opnd[1][s], it)
                if codes:
                    for c in range(2):
                        assert bhalf[c][s] == [it] * group_warps, ("B half", c, bhalf[c][s], it)
                in_use[s] = it
                consumed.append(it)

                def release(s=s):
                    in_use[s] = None
                    empty[0][s].arrive()
                    if multicast_empty:
                        empty[1][s].arrive()
                commits.append(release)
                it += 1

            def finish(buf=buf, local=local):
                for c in range(2):
                    dbuf[c][buf] = (local, True)
                    tfull[c][buf].arrive()
            commits.append(finish)

    def epilogue(c):
        for local in range(ntiles):
            buf = local & 1
            yield lambda buf=buf, local=local: tfull[c][buf].done((local >> 1) & 1)
            assert dbuf[c][buf] == (local, True), ("epilogue", c, dbuf[c][buf], local)
            reads[c][buf] += 1
            tempty[buf].arrive()

    actors = [producer(0), producer(1), mma()] + [epilogue(c) for c in range(2) for _ in range(EPI)]
    if codes:
        actors += [decoder(c, g, w) for c in range(2) for g in range(groups) for w in range(group_warps)]
        actors += [forwarder()]
    waits = [None] * len(actors)
    alive = list(range(len(actors)))
    while alive or landings or commits:
        ready = [("step", i) for i in alive if waits[i] is None or waits[i]()]
        ready += [("land", j) for j in range(len(landings))]
        ready += [("commit", 0)] if commits else []
        assert ready, f"deadlock: {ntiles} tiles x {kblocks} k-blocks"
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
    rng = random.Random(3 * n)
    for seed in range(n):
        yield rng.randint(1, 4), rng.choice([1, 2, 3, 4, 7, 16]), seed


# (decoder groups, warps per group): the decode form at d = 8 with 8 decoder
# warps is one group of 8; the other coded kinds with 8 warps are two groups of 4
@pytest.mark.parametrize("groups,group_warps", [(1, 8), (2, 4)])
def test_pair_protocol_with_codes(groups, group_warps):
    for ntiles, kblocks, seed in _cases(60):
        run(ntiles, kblocks, groups, group_warps, True, seed)


def test_pair_protocol_without_codes():
    """dW: both operands by copy, no decoders and no handover."""
    for ntiles, kblocks, seed in _cases(60):
        run(ntiles, kblocks, 1, 1, False, seed)


@pytest.mark.parametrize("mutation", [
    dict(multicast_empty=False),      # stage release committed to the even CTA only
    dict(tempty_count=EPI),           # accumulator released by one CTA's epilogue warps
    dict(mma_waits_peer=False),       # the odd CTA's B half taken without the handover
    dict(forward_at_first=True),      # the handover sent at a group's first k-block
])
def test_the_model_catches_a_broken_pair_protocol(mutation):
    caught = False
    for ntiles, kblocks, seed in _cases(60):
        try:
            run(ntiles, kblocks, 2, 4, True, seed, **mutation)
        except AssertionError:
            caught = True
            break
    assert caught
