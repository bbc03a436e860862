"""The ordering protocol of the row-parallel group, as a model on CPU.

The device words of spear_w4ec_tp_* (csrc/tp.cu): per rank p a count of
completed calls, and in every rank's buffer one ready word and one done word
per rank.  Per call c (counted from 1) rank p runs, in stream order:
  push    waits until done[q] >= c - 1 in its own buffer for every q, then
          writes its u partial of call c into slot p of every rank's buffer;
  forward writes its partial output of call c into its own buffer;
  signal  sets ready[p] = c in every rank's buffer;
  reduce  waits until ready[q] >= c in its own buffer for every q, reads its
          u slots and every rank's partial output, then sets done[p] = c in
          every rank's buffer and its count to c.
This model runs those steps for several ranks and calls under random
schedules (any rank may move whenever its next step is not blocked) and
checks that every read sees the data of its own call (no overwrite before
the read, no stale data) and that no schedule deadlocks.  It checks the
design of the words, not the kernels (those are checked on the GPU).
"""
from __future__ import annotations

import random

import pytest

STEPS = ("push", "forward", "signal", "reduce")


def _run(world: int, calls: int, seed: int, drop_wait: str | None = None):
    rng = random.Random(seed)
    ready = [[0] * world for _ in range(world)]    # ready[owner][q]
    done = [[0] * world for _ in range(world)]     # done[owner][q]
    slots = [[None] * world for _ in range(world)]  # slots[owner][q]: call of rank q's u partial held there
    ypart = [None] * world                           # call of each rank's partial output
    pos = [(1, 0)] * world                           # (call, step index) of each rank
    errors = []

    def blocked(p):
        c, i = pos[p]
        if c > calls:
            return True
        step = STEPS[i]
        if step == "push" and drop_wait != "done":
            return any(done[p][q] < c - 1 for q in range(world))
        if step == "reduce" and drop_wait != "ready":
            return any(ready[p][q] < c for q in range(world))
        return False

    while any(pos[p][0] <= calls for p in range(world)):
        movable = [p for p in range(world) if not blocked(p)]
        if not movable:
            return "deadlock", errors
        p = rng.choice(movable)
        c, i = pos[p]
        step = STEPS[i]
        if step == "push":
            for q in range(world):
                slots[q][p] = c
        elif step == "forward":
            ypart[p] = c
        elif step == "signal":
            for q in range(world):
                ready[q][p] = c
        else:
            for q in range(world):
                if slots[p][q] != c:
                    errors.append(("u slot", p, q, c, slots[p][q]))
                if ypart[q] != c:
                    errors.append(("partial output", p, q, c, ypart[q]))
            for q in range(world):
                done[q][p] = c
        pos[p] = (c + 1, 0) if i == len(STEPS) - 1 else (c, i + 1)
    return "finished", errors


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_every_schedule_reads_its_own_call_and_finishes(world):
    for seed in range(300):
        state, errors = _run(world, calls=6, seed=seed)
        assert state == "finished", (world, seed)
        assert not errors, (world, seed, errors[:3])


@pytest.mark.parametrize("dropped", ["done", "ready"])
def test_each_wait_is_needed(dropped):
    """Planted mistake: without the wait for the done words a fast rank
    overwrites what a slow rank still has to read; without the wait for the
    ready words a rank reads partials of an earlier call.  Some schedule
    shows it."""
    found = False
    for seed in range(300):
        state, errors = _run(3, calls=4, seed=seed, drop_wait=dropped)
        if errors:
            found = True
            break
    assert found
