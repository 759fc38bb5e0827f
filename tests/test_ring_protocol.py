"""A randomised model of the bulk dispatch kernel's shared-memory ring (CPU only).

The kernel (``dispatch_kernel`` in csrc/ep_dispatch.cu) runs one warp per CTA over its units
i = 0 .. n-1 with an S-stage ring:

- prologue: units 0 .. min(S, n)-1 are loaded into stages 0 .. S-1, each completing the stage's
  mbarrier once;
- unit i: wait on stage i mod S's mbarrier for phase parity (i / S) mod 2, issue the bulk stores
  that read the stage, commit them as one group;
- then, if 1 <= i and i - 1 + S < n: wait until every group but the newest has finished reading
  shared memory (``cp.async.bulk.wait_group.read 1``) and load unit i - 1 + S into stage
  (i - 1) mod S.

The model replays that schedule with random load latencies and store read durations and checks
that it is race-free and live for every ring depth the launch rules produce (2 .. 16 stages,
the 3-stage rings of the normal-mode dispatch at 4 CTAs per SM included) and for unit counts
below, at and far above the ring size:

- each wait finds its own unit's fill (never a stale one, never one two phases ahead, which a
  parity wait could not tell apart) and never waits on a fill that was not issued (a deadlock);
- no load is issued into a stage that a store group is still reading;
- every unit is consumed exactly once, in order.
"""
import random

import pytest


def run_ring(S: int, n: int, rng: random.Random, lag: int = 1, wait_reads: bool = True):
    """Replay the schedule; `lag` = 1 and `wait_reads` are the kernel's (refill the stage of unit
    i - lag after ``wait_group.read 1``); other values plant a mistake for the model to catch."""
    clock = 0.0
    fills = {s: [] for s in range(S)}      # stage -> [(unit, issue time, landing time)]
    reads = {}                              # group (= unit) -> (stage, read start, read end)
    consumed = []

    def issue(unit):
        s = unit % S
        for g, (gs, _, end) in reads.items():
            assert not (gs == s and end > clock), f"S={S} n={n}: unit {unit} loaded over stage {s} " \
                                                  f"while group {g} still reads it"
        fills[s].append((unit, clock, clock + rng.expovariate(1.0)))

    for i in range(min(S, n)):
        issue(i)
    for i in range(n):
        s = i % S
        parity_phase = i // S                       # the fill this wait must see: number i // S of stage s
        assert len(fills[s]) > parity_phase, f"S={S} n={n}: unit {i} waits on a fill never issued"
        unit, _, landed = fills[s][parity_phase]
        assert unit == i, f"S={S} n={n}: stage {s} phase {parity_phase} holds unit {unit}, not {i}"
        clock = max(clock, landed)
        # a parity wait cannot tell phase p from p + 2: no later fill of this stage may have landed
        later = [f for f in fills[s][parity_phase + 1:] if f[2] <= clock]
        assert not later, f"S={S} n={n}: stage {s} refilled before unit {i} was consumed"
        consumed.append(i)
        reads[i] = (s, clock, clock + rng.expovariate(2.0))
        refill = i - lag + S
        if i >= lag and refill < n:
            if wait_reads:
                # wait_group.read 1: every group but the newest (i) has finished reading
                clock = max([clock] + [end for g, (_, _, end) in reads.items() if g <= i - 1])
            issue(refill)
    # bulk_wait 0 at exit: all stores done; every unit consumed once, in order
    assert consumed == list(range(n))
    assert all(len(fills[s]) == len([u for u in range(n) if u % S == s]) for s in range(S))


@pytest.mark.parametrize("S", list(range(2, 17)))
def test_ring_is_race_free_and_live(S):
    rng = random.Random(1000 + S)
    for n in sorted({0, 1, S - 1, S, S + 1, 2 * S - 1, 2 * S, 2 * S + 1, 7 * S + 3, 97}):
        for _ in range(40):
            run_ring(S, n, rng)


@pytest.mark.parametrize("lag,wait_reads", [(0, True), (1, False)])
def test_model_catches_a_broken_schedule(lag, wait_reads):
    """Planted mistakes: refilling the stage of the unit just consumed (whose stores the read wait
    does not cover), or refilling without the read wait.  Both overwrite a stage that a store may
    still be reading, and the model must say so."""
    rng = random.Random(7)
    with pytest.raises(AssertionError, match="still reads it"):
        for _ in range(50):
            run_ring(4, 40, rng, lag=lag, wait_reads=wait_reads)
