"""A host-side model of the stream order under programmatic dependent launch
(PDL) that the decode-GEMV relies on (include/lcvq.h, "Stream order under
programmatic dependent launch"), run under random interleavings.

A stream holds kernels in order.  A kernel launched with PDL may start once
its predecessor has triggered (griddepcontrol.launch_dependents; a kernel
that never triggers does so when it finishes); one launched without PDL starts
once its predecessor's writes are visible.  A finished kernel's writes become
visible some time later (modelled as a separate event); griddepcontrol.wait
returns only once the predecessor has finished and its writes are visible, and
every kernel here waits (or is launched without PDL) before it finishes, so
after a wait every earlier kernel's writes are visible.  Reads before the wait
have no such guarantee.

Kernels of a QAT-then-decode sequence:
- assign_pack (no PDL): writes the packed codes, finishes;
- the X-transform (PDL): waits, then triggers, then writes X'' and finishes;
- the decode-GEMV (PDL): when it follows its X-transform it reads the codes
  before its wait ("early codes"), otherwise after; it reads X'' after its
  wait, then finishes;
- lcvq_gemm_xformed's GEMV (PDL, no X-transform in front): waits first.

The model checks the two rules that make the early code reads safe: a GEMV
reads the codes only once every earlier code write is visible, and X'' only
once the X-transform's writes are.  It also shows what breaks them: an
X-transform that triggers before its wait, or a GEMV that reads codes early
without an X-transform in front of it (the kernel before it may have finished
without its writes being visible yet).
"""

import random

import pytest


def run(stream, seed):
    """stream: list of (kind, options) with kind in {"pack", "xform", "gemv"}."""
    rng = random.Random(seed)
    n = len(stream)
    state = ["queued"] * n            # queued -> running -> finished -> visible
    triggered = [False] * n
    xpp_ready = set()                 # X-transforms whose output is visible

    def code_writes_pending(i):  # a code writer before i whose writes are not visible yet
        return any(stream[j][0] == "pack" and state[j] != "visible" for j in range(i))

    def can_start(i):
        if i == 0:
            return True
        pdl = stream[i][0] != "pack"
        return state[i - 1] == "visible" or (pdl and triggered[i - 1])

    def waited(i):  # griddepcontrol.wait
        return i == 0 or state[i - 1] == "visible"

    def body(i):
        kind, opt = stream[i]
        if kind == "xform":
            if opt.get("trigger_first"):
                triggered[i] = True
            yield lambda: waited(i)
            triggered[i] = True
        elif kind == "gemv":
            early = opt.get("early", False)
            if early:
                assert not code_writes_pending(i), "codes read before their writes are visible"
            yield lambda: waited(i)
            if not early:
                assert not code_writes_pending(i), "codes read before their writes are visible"
            src = opt.get("xpp_from")
            if src is not None:
                assert src in xpp_ready, "X'' read before the X-transform's writes are visible"
        yield None

    gens = [None] * n
    waits = [None] * n
    while any(st != "visible" for st in state):
        ready = []
        for i in range(n):
            if state[i] == "queued" and can_start(i):
                ready.append(("start", i))
            elif state[i] == "running" and (waits[i] is None or waits[i]()):
                ready.append(("step", i))
            elif state[i] == "finished":
                ready.append(("flush", i))
        assert ready, "deadlock"
        kind, i = rng.choice(ready)
        if kind == "start":
            state[i] = "running"
            gens[i] = body(i)
            waits[i] = None
        elif kind == "flush":
            state[i] = "visible"
            if stream[i][0] == "xform":
                xpp_ready.add(i)
        else:
            try:
                waits[i] = next(gens[i])
            except StopIteration:
                state[i] = "finished"
                triggered[i] = True


def _qat_then_decode(trigger_first=False, early_without_xform=False):
    s = [("pack", {}),
         ("xform", {"trigger_first": trigger_first}),
         ("gemv", {"early": True, "xpp_from": 1}),
         ("pack", {}),
         ("xform", {"trigger_first": trigger_first}),
         ("gemv", {"early": True, "xpp_from": 4}),
         ("gemv", {"early": early_without_xform, "xpp_from": 4})]   # lcvq_gemm_xformed
    return s


def test_early_code_reads_are_safe_in_the_library_order():
    for seed in range(400):
        run(_qat_then_decode(), seed)


def test_an_x_transform_that_triggers_before_its_wait_breaks_it():
    failures = 0
    for seed in range(400):
        try:
            run(_qat_then_decode(trigger_first=True), seed)
        except AssertionError:
            failures += 1
    assert failures > 0


def test_early_code_reads_without_an_x_transform_in_front_break_it():
    stream = [("pack", {}), ("gemv", {"early": True})]
    failures = 0
    for seed in range(400):
        try:
            run(stream, seed)
        except AssertionError:
            failures += 1
    assert failures > 0
