"""A host-side model of the CTA-pair decode form's barrier protocol in
csrc/tc_gemm.cu (tc2_gemm_kernel with codes), run under random interleavings.

Roles, one step at a time:
- each CTA's decoders fill ring slot s with k block `it` once the MMA has
  released the slot (empty[s]), then arrive on their CTA's decd[s];
- the odd CTA's forwarder waits for its decd[s] and, at the end of every group
  of G k blocks (or at the very last one), arrives once on the even CTA's
  decd_peer[(it / G) % S];
- the even CTA's MMA issuer waits for its own decd[s] and, at the first k block
  of a group, for decd_peer[q % S] in phase (q / S) & 1.  It then consumes
  both CTAs' slot s and releases it on both CTAs' empty[s].

The barriers follow mbarrier phase semantics: an arrival count per phase, and a
parity wait that passes once the phase of that parity has completed.  The model
checks three properties:
- every k block is consumed in order, with both slots holding exactly that k block;
- no barrier receives an arrival for a phase nobody has waited out (no parity aliasing);
- nothing deadlocks.
"""

import random

import pytest


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.phase = count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count

    def done(self, parity):  # try_wait.parity: the phase with this parity has completed
        return (self.phase & 1) != parity


def run(S, G, total, seed, early=False):
    rng = random.Random(seed)
    empty = [[Bar(1) for _ in range(S)] for _ in range(2)]
    decd = [[Bar(1) for _ in range(S)] for _ in range(2)]
    peer = [Bar(1) for _ in range(S)]
    slot = [[None] * S for _ in range(2)]
    consumed = []
    peer_waited = [0] * S  # phases of decd_peer[b] the MMA has waited out

    def decoder(c):
        for it in range(total):
            s, ph = it % S, (it // S) & 1
            yield lambda: empty[c][s].done(ph ^ 1)
            slot[c][s] = it
            decd[c][s].arrive()

    def forwarder():
        for it in range(total):
            s, ph = it % S, (it // S) & 1
            yield lambda: decd[1][s].done(ph)
            if it % G == (0 if early else G - 1) or it == total - 1:
                b = (it // G) % S
                # the phase this arrival completes must be the next one the MMA waits for
                assert peer[b].phase == peer_waited[b], "decd_peer phase aliasing"
                peer[b].arrive()

    def mma():
        for it in range(total):
            s, ph = it % S, (it // S) & 1
            yield lambda: decd[0][s].done(ph)
            if it % G == 0:
                q = it // G
                b = q % S
                yield lambda: peer[b].done((q // S) & 1)
                peer_waited[b] += 1
            # the odd CTA's slot is complete only if its whole group was forwarded
            assert slot[0][s] == it and slot[1][s] == it, (it, slot[0][s], slot[1][s])
            consumed.append(it)
            empty[0][s].arrive()
            empty[1][s].arrive()

    actors = [decoder(0), decoder(1), forwarder(), mma()]
    waits = [next(a) for a in actors]
    alive = [True] * len(actors)
    while any(alive):
        ready = [i for i, a in enumerate(actors) if alive[i] and waits[i]()]
        assert ready, f"deadlock at S={S} G={G} total={total}: consumed {len(consumed)}"
        i = rng.choice(ready)
        try:
            waits[i] = next(actors[i])
        except StopIteration:
            alive[i] = False
    assert consumed == list(range(total))


@pytest.mark.parametrize("G", [1, 2, 3, 4, 5])
def test_grouped_handover_is_safe_for_every_group_size_below_the_ring(G):
    for total in (1, 2, 3, 5, 6, 7, 64, 257, 320):
        for seed in range(6):
            run(6, G, total, seed)


def test_a_group_longer_than_the_ring_deadlocks():
    """A group of S + 1 k blocks needs a slot decoded twice before its first k
    block is consumed, and a slot comes back only once it is consumed, so the
    model stalls.  The kernel keeps G < S: at G = S the protocol still holds,
    but each group drains the ring."""
    run(6, 6, 64, 0)
    with pytest.raises(AssertionError, match="deadlock"):
        run(6, 7, 64, 0)


def test_the_model_catches_a_handover_sent_too_early():
    """A forwarder that arrives at the first k block of its group instead of
    the last lets the MMA take odd-CTA slots that are not decoded yet."""
    failures = 0
    for seed in range(20):
        try:
            run(6, 3, 64, seed, early=True)
        except AssertionError:
            failures += 1
    assert failures > 0
