"""A model of the stage ring the GEMV kernels run, checked on the CPU.

One producer fills ns slots in stage order (it waits for a slot's `empty`
barrier before reusing it); the bulk copies land in any order; two consumer
groups take alternate stages, each waiting on the slot's `full` barrier by
phase parity and then arriving on its `empty` barrier.  An mbarrier's
parity wait passes when the phase of that parity among the current and the
previous one has completed, so it cannot tell phase k from phase k + 2.

The model explores random schedules and checks that a group only consumes
a stage whose copy has landed and not been overwritten.  With an odd ring
depth a slot alternates between the groups, and without the kernels'
release wait (a group first waits for the other group's release of the
slot) some schedule breaks that; with it, no schedule does, at any depth.
"""
import random

import pytest


class Barrier:
    def __init__(self):
        self.completed = 0          # phases completed so far

    def passes(self, parity):       # try_wait.parity
        return (self.completed & 1) != parity


def run(ns, release_wait, stages, rng):
    full = [Barrier() for _ in range(ns)]
    empty = [Barrier() for _ in range(ns)]
    empty_arrivals = [0] * ns       # arrivals towards the current phase (one per group release)
    slot_holds = [None] * ns        # the stage whose bytes the slot holds
    issued, in_flight = 0, []
    nxt = [0, 1]                    # next stage of each group
    while nxt[0] < stages or nxt[1] < stages:
        moves = []
        if issued < stages:
            k = issued
            s, ph = k % ns, (k // ns) & 1
            if k < ns or empty[s].passes(ph ^ 1):
                moves.append(("issue", k))
        moves += [("land", k) for k in in_flight]
        for g in (0, 1):
            k = nxt[g]
            if k >= stages:
                continue
            s, ph = k % ns, (k // ns) & 1
            if release_wait and ns % 2 == 1 and k >= ns and not empty[s].passes(ph ^ 1):
                continue
            if full[s].passes(ph):
                moves.append(("consume", g))
        if not moves:
            raise AssertionError("deadlock")
        kind, v = rng.choice(moves)
        if kind == "issue":
            issued += 1
            in_flight.append(v)
        elif kind == "land":
            in_flight.remove(v)
            slot_holds[v % ns] = v
            full[v % ns].completed += 1
        else:
            g = v
            k = nxt[g]
            s = k % ns
            if slot_holds[s] != k:
                return False        # consumed a stage that is not (or no longer) in its slot
            empty_arrivals[s] += 1
            if empty_arrivals[s] == 1:   # one arrival stands for the group's 8 warps
                empty_arrivals[s] = 0
                empty[s].completed += 1
            nxt[g] += 2
    return True


@pytest.mark.parametrize("ns", [2, 3, 4, 5, 7, 8])
def test_release_wait_makes_every_depth_safe(ns):
    rng = random.Random(1000 + ns)
    for _ in range(3000):
        assert run(ns, True, 4 * ns + 3, rng)


@pytest.mark.parametrize("ns", [2, 4, 6, 8])
def test_even_depth_is_safe_without_it(ns):
    rng = random.Random(2000 + ns)
    for _ in range(3000):
        assert run(ns, False, 4 * ns + 3, rng)


@pytest.mark.parametrize("ns", [3, 5])
def test_odd_depth_without_it_can_read_a_stage_that_has_not_landed(ns):
    rng = random.Random(3000 + ns)
    assert any(not run(ns, False, 4 * ns + 3, rng) for _ in range(20000))
