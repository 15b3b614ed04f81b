"""Host model of the batched expert kernels' copy schedule (the per-warp ring
of kSlots steps filled with asynchronous copies, one commit group per step).

The model replays the order in which one warp issues, commits, waits for and
consumes steps across a sequence of segments -- including segments in which
the warp owns no steps and steps whose refill crosses into the next segment
-- and checks the invariant the kernel relies on: after waiting until at most
kSlots-1 groups are pending, the slot of the step about to be computed holds
that step's completed copy, and no slot is refilled before its step is used.
"""
import random

import pytest

K_SLOTS = 3  # qe_grouped.cu kSlots


class Ring:
    def __init__(self, n):
        self.slot = [None] * n        # completed contents
        self.consumed = [True] * n    # the slot's last completed step was used
        self.pending = []             # groups: list of (slot, tag)
        self.open = []                # copies issued since the last commit
        self.inflight = set()         # slots targeted by pending copies

    def issue(self, j, tag):
        assert j not in self.inflight, "slot refilled while a copy into it is pending"
        assert self.consumed[j], "slot refilled before its step was used"
        self.open.append((j, tag))
        self.inflight.add(j)

    def commit(self):
        self.pending.append(self.open)
        self.open = []

    def wait(self, n):
        while len(self.pending) > n:
            for j, tag in self.pending.pop(0):
                self.slot[j] = tag
                self.consumed[j] = False
                self.inflight.discard(j)

    def consume(self, j, tag):
        assert j not in self.inflight and self.slot[j] == tag, (j, self.slot[j], tag)
        self.consumed[j] = True


def run_warp(steps):
    """steps[s] = steps this warp owns in segment s (0 allowed)."""
    ring = Ring(K_SLOTS)
    done = []
    for j in range(K_SLOTS):  # the kernel's initial fill of segment 0
        if j < steps[0]:
            ring.issue(j, (0, j))
        ring.commit()
    for s, nst in enumerate(steps):
        nstp = -(-nst // K_SLOTS) * K_SLOTS
        nst_n = steps[s + 1] if s + 1 < len(steps) else 0
        for l0 in range(0, nstp, K_SLOTS):
            for j in range(K_SLOTS):
                l = l0 + j
                ring.wait(K_SLOTS - 1)
                if l < nst:
                    ring.consume(j, (s, l))
                    done.append((s, l))
                ln = l + K_SLOTS
                if ln < nst:
                    ring.issue(j, (s, ln))
                elif ln >= nstp and ln - nstp < nst_n:
                    ring.issue(j, (s + 1, ln - nstp))
                ring.commit()
        if nstp == 0:
            for j in range(K_SLOTS):
                if j < nst_n:
                    ring.issue(j, (s + 1, j))
                ring.commit()
    ring.wait(0)
    return done


@pytest.mark.parametrize("seed", range(40))
def test_every_step_reads_its_own_completed_copy(seed):
    rng = random.Random(seed)
    n = rng.randint(1, 12)
    # unit counts of the real shapes (4 per warp at 128/256-row items, 8 or 16
    # for down) times chunks per lane, plus warps with no unit at all
    choices = [0, 1, 2, 3, 4, 5, 8, 16, 32, 7]
    steps = [rng.choice(choices) for _ in range(n)]
    done = run_warp(steps)
    assert done == [(s, l) for s, nst in enumerate(steps) for l in range(nst)]


def test_segments_without_steps_between_busy_ones():
    steps = [0, 5, 0, 0, 3, 1, 0, 4]
    done = run_warp(steps)
    assert done == [(s, l) for s, nst in enumerate(steps) for l in range(nst)]
