"""A host-side model of the stage ring of the wide-tile decode-GEMV in
csrc/gemv.cu (gemv_wide_kernel: large groups at M <= 16, bf16 and int8), run
under random interleavings, with the byte counts of every copy.

The producer warp, per K chunk c (512 positions) of each tile, waits for
empty[s] in phase ((seq / S) & 1) ^ 1 and arms full[s] with the chunk's bytes:
one 128-row x 128-byte code box (counted whole, zero fill included) plus
M * xbytes of activations, xbytes = 2 * min(512, K - 512 c); it then starts
the code box and the activation copies -- bf16: one copy of xbytes per token;
int8: one copy of xbytes / 2 per token and digit plane.  The eight consumer
warps wait for full[s] in phase (seq / S) & 1 and arrive on empty[s].  At the
end the producer drains: it waits for the release of the next S stages.

Each copy lands separately, in any order.  The model checks that a stage's
full phase completes exactly when the last of its copies has landed (the
armed byte count equals the bytes copied, for every M, path and K tail), that
no copy overwrites a stage a consumer still reads, that every consumer reads
its own chunk, and that nothing deadlocks, the drain included.
"""

import random

import pytest

CONSUMERS = 8
CODE_BYTES = 128 * 128


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
        assert self.tx >= 0, "more bytes landed than the phase was armed with"
        self._advance()

    def done(self, parity):
        return (self.phase & 1) != parity


def chunk_copies(K, c, M, int8):
    """Byte counts of the copies the producer starts for chunk c."""
    xk = 512 * c
    xbytes = (K - xk) * 2 if K - xk < 512 else 1024
    if int8:
        x = [xbytes // 2] * (2 * M)
    else:
        x = [xbytes] * M
    return CODE_BYTES + M * xbytes, [CODE_BYTES] + x


def run(Ks, M, int8, S, seed, armed_extra=0):
    rng = random.Random(seed)
    full = [Bar(1) for _ in range(S)]
    empty = [Bar(CONSUMERS) for _ in range(S)]
    stage = [None] * S        # (chunk seq, copies landed, copies total)
    readers = [0] * S         # consumers reading the stage's current chunk
    landings = []
    chunks = [(t, c) for t, K in enumerate(Ks) for c in range(-(-K // 512))]

    def producer():
        seq = 0
        for t, c in chunks:
            s = seq % S
            yield lambda s=s, seq=seq: empty[s].done(((seq // S) & 1) ^ 1)
            armed, copies = chunk_copies(Ks[t], c, M, int8)
            assert readers[s] == 0, "stage refilled while a consumer reads it"
            full[s].arrive_expect_tx(armed + armed_extra)
            stage[s] = [seq, 0, len(copies)]
            for nbytes in copies:
                def land(s=s, nbytes=nbytes, seq=seq):
                    assert stage[s][0] == seq
                    stage[s][1] += 1
                    before = full[s].phase
                    full[s].complete_tx(nbytes)
                    if full[s].phase != before:  # the phase completed with this copy
                        assert stage[s][1] == stage[s][2], "stage marked full before its last copy"
                landings.append(land)
            seq += 1
        for _ in range(S):  # the drain
            s = seq % S
            yield lambda s=s, seq=seq: empty[s].done(((seq // S) & 1) ^ 1)
            seq += 1

    def consumer():
        for seq in range(len(chunks)):
            s = seq % S
            yield lambda s=s, seq=seq: full[s].done((seq // S) & 1)
            assert stage[s][0] == seq and stage[s][1] == stage[s][2], (seq, stage[s])
            readers[s] += 1
            yield None  # the MMAs over the stage
            readers[s] -= 1
            empty[s].arrive()

    actors = [producer()] + [consumer() for _ in range(CONSUMERS)]
    waits = [None] * len(actors)
    alive = list(range(len(actors)))
    while alive or landings:
        ready = [("step", i) for i in alive if waits[i] is None or waits[i]()]
        ready += [("land", j) for j in range(len(landings))]
        assert ready, f"deadlock: K {Ks}, M {M}, int8 {int8}"
        kind, i = rng.choice(ready)
        if kind == "land":
            landings.pop(i)()
        else:
            try:
                waits[i] = next(actors[i])
            except StopIteration:
                alive.remove(i)


@pytest.mark.parametrize("int8,Ms,S", [(True, [1, 2, 3, 4], 4), (False, [1, 5, 8], 4),
                                        (False, [9, 13, 16], 6)])
def test_ring_bytes_and_phases_for_every_token_count_and_k_tail(int8, Ms, S):
    rng = random.Random(11)
    for M in Ms:
        for trial in range(25):
            Ks = [64 * rng.randint(1, 40) for _ in range(rng.randint(1, 3))]  # every K tail
            run(Ks, M, int8, S, seed=1000 * M + trial)


def test_the_model_catches_a_wrong_byte_count():
    """A stage armed with 16 bytes more than its copies bring never completes."""
    with pytest.raises(AssertionError, match="deadlock"):
        run([1088], 3, True, 4, seed=0, armed_extra=16)
