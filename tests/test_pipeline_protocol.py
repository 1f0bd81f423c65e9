"""Model of the small-batch kernel's shared-memory ring protocol (producer
thread, helper warps, consumer warps) with mbarrier parity waits, run under
random interleavings on the CPU.

An mbarrier wait names only the parity of the phase it waits for, so a waiter
that reaches phase k of a slot before phase k-1 of that slot is known complete
passes at once on stale data.  The kernel therefore gives a helper fixed ring
slots (the helper count divides the ring depth).  This test checks that every
configuration the host launches completes with every chunk processed on its
own data, and that the rotating assignment the kernel excludes does not.
"""
import random

import pytest


def _run(nit, stages, nh, seed):
    """'ok', or a description of a deadlock or a stale read."""
    rnd = random.Random(seed)
    full = [0] * stages      # completed phases of each slot's TMA barrier
    sxful = [0] * stages     # completed phases of the helper -> consumer barrier
    empty = [0] * stages     # completed phases of the consumer -> producer barrier
    ready = lambda bar, s, parity: (bar[s] & 1) != parity  # mbarrier try_wait.parity
    prod_c, landing, cons_c = 0, [], 0
    help_c = list(range(nh))
    sx_chunk = [None] * stages   # chunk whose activations the helper left in a slot
    while True:
        progressed = False
        actors = ["producer", "tma", "consumers"] + [("helper", h) for h in range(nh)]
        rnd.shuffle(actors)
        for a in actors:
            if a == "producer" and prod_c < nit:
                s, ph = prod_c % stages, (prod_c // stages) & 1
                if prod_c < stages or ready(empty, s, ph ^ 1):
                    landing.append((s, prod_c))
                    prod_c += 1
                    progressed = True
            elif a == "tma" and landing:
                s, c = landing.pop(rnd.randrange(len(landing)))
                full[s] += 1
                progressed = True
            elif a == "consumers" and cons_c < nit:
                s, ph = cons_c % stages, (cons_c // stages) & 1
                if ready(sxful, s, ph):
                    if sx_chunk[s] != cons_c:
                        return f"stale: consumers read chunk {sx_chunk[s]} as {cons_c}"
                    empty[s] += 1
                    cons_c += 1
                    progressed = True
            elif isinstance(a, tuple):
                h = a[1]
                c = help_c[h]
                if c < nit:
                    s, ph = c % stages, (c // stages) & 1
                    if ready(full, s, ph):
                        if full[s] != c // stages + 1:
                            return f"stale: helper {h} took chunk {c} before it landed"
                        sx_chunk[s] = c
                        sxful[s] += 1
                        help_c[h] = c + nh
                        progressed = True
        if cons_c == nit:
            return "ok"
        if not progressed:
            return f"deadlock: produced {prod_c}, consumed {cons_c}, helpers at {help_c}"


def _helpers_launched(B, stages):
    """The host's choice (run_gemv in q4_api.cu) and the kernel's guard."""
    nl = 2 if (B >= 4 and stages % 2 == 0) else 1
    return nl if stages % nl == 0 else 1


@pytest.mark.parametrize("stages", [2, 3, 4])
@pytest.mark.parametrize("B", [1, 4, 8])
def test_launched_configurations_are_safe(stages, B):
    nh = _helpers_launched(B, stages)
    for nit in [1, 2, 3, 5, 8, 13, 24, 25, 50]:
        for seed in range(150):
            assert _run(nit, stages, nh, seed) == "ok", (nit, stages, nh, seed)


def test_rotating_helpers_are_unsafe():
    """Two helpers over a ring of three slots: some interleaving reads stale
    data or deadlocks -- the reason the kernel forbids it."""
    results = {_run(nit, 3, 2, seed) for nit in [5, 8, 13] for seed in range(200)}
    assert any(r != "ok" for r in results)
