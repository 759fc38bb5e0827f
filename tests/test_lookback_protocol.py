"""A randomised model of the one-launch look-back layout's cross-CTA protocol (CPU only).

``layout_lookback_kernel`` (csrc/ep_layout.cu) keeps its barrier state in the first 64 KiB of the
caller's workspace from call to call: an epoch word, then one flag word per chunk, 32 words apart.
Per call, CTA (chunk) g:

1. reads the epoch E_g and sets value = 2 (E_g + 1);
2. writes its chunk histogram, then release-stores value into flag 32 g;
3. waits (bounded) until the flag of every chunk g' < g holds at least value, then sums their
   histograms;
4. if g is the last chunk, advances the epoch to max(epoch, E_g + 1), whether or not its wait
   passed.

The fused cooperative path shares the region: every CTA reads the epoch, stores 2 (E + 1) and
then 2 (E + 1) + 1 into flag g (contiguous words), and advances the epoch to E + 1.

The model schedules CTAs in launch order onto a limited number of resident slots, lets any
resident CTA step at random, and checks that a waiting CTA only ever accepts flags (and so
histograms) that its own call wrote, across long random sequences of both paths with different
chunk counts.  It also records the one case the scheme does not cover: after a wait has given up
(EP_STATUS_TIMEOUT), a chunk that read the epoch only after the last chunk advanced it leaves a
flag the next call accepts, unless the caller zero-fills the region again, as the header asks.
"""
import random

import pytest

STRIDE = 32


class Region:
    def __init__(self):
        self.epoch = 0
        self.flags = {}     # word index -> value
        self.hist = {}      # chunk -> call id of the histogram last written there

    def flag(self, i):
        return self.flags.get(i, 0)


def lookback_call(ws, G, call, rng, resident, spin_limit=10 ** 9, stall=None):
    """One call; returns (stale acceptances, timed out).  `stall` = (chunk, steps): that chunk,
    once resident, does nothing for that many of its turns before reading the epoch."""
    state = ["pending"] * G
    epoch_of, spins, stalled = [0] * G, [0] * G, [0] * G
    seen = [0] * G          # a waiting chunk's predecessors below this index have been seen
    stale, timed_out = [], False
    live, nxt, done = [], 0, 0
    while done < G:
        while nxt < G and len(live) < resident:          # dispatch in launch order
            state[nxt] = "resident"
            if stall and stall[0] == nxt:
                stalled[nxt] = stall[1]
            live.append(nxt)
            nxt += 1
        g = live[rng.randrange(len(live))]
        st = state[g]
        finished = False
        if st == "resident":
            if stalled[g] > 0:
                stalled[g] -= 1
                continue
            epoch_of[g] = ws.epoch
            state[g] = "read"
        elif st == "read":
            ws.hist[g] = call
            ws.flags[STRIDE * g] = 2 * (epoch_of[g] + 1)
            state[g] = "wait"
        else:                                                # waiting on chunks 0 .. g-1
            value = 2 * (epoch_of[g] + 1)
            while seen[g] < g and ws.flag(STRIDE * seen[g]) >= value:
                seen[g] += 1                                 # flags only grow: a seen flag stays seen
            if seen[g] == g:
                stale += [(g, p) for p in range(g) if ws.hist.get(p) != call]
                finished = True
            else:
                spins[g] += 1
                if spins[g] >= spin_limit:                   # the bounded wait gives up
                    timed_out = True
                    finished = True
            if finished and g == G - 1:
                ws.epoch = max(ws.epoch, epoch_of[g] + 1)
        if finished:
            state[g] = "done"
            live.remove(g)
            done += 1
    return stale, timed_out


def fused_call(ws, G):
    e = ws.epoch
    for g in range(G):
        ws.flags[g] = 2 * (e + 1)
    for g in range(G):
        ws.flags[g] = 2 * (e + 1) + 1
    ws.epoch = max(ws.epoch, e + 1)


def test_no_call_accepts_another_calls_flags():
    rng = random.Random(11)
    ws = Region()
    for call in range(1500):
        if rng.random() < 0.2:
            fused_call(ws, rng.randint(1, 255))
            continue
        G = rng.randint(1, 255)
        stale, timed_out = lookback_call(ws, G, call, rng, resident=rng.randint(1, G))
        assert not timed_out and not stale, (call, G, stale)


def test_a_timeout_can_poison_the_next_call_unless_the_region_is_zeroed():
    """Chunk 1 stalls before reading the epoch for longer than the last chunk's wait limit: the
    last chunk gives up and advances the epoch, chunk 1 then reads the new epoch and leaves a flag
    at the next call's value.  Without zero-filling, the next call's chunk 2 accepts it while chunk
    1 of that call has not written its histogram yet; after zero-filling it cannot."""
    found = False
    for seed in range(200):
        rng = random.Random(seed)
        ws = Region()
        _, timed_out = lookback_call(ws, 3, 0, rng, resident=3, spin_limit=5, stall=(1, 60))
        if not timed_out:
            continue
        poisoned = Region()
        poisoned.__dict__.update({k: (dict(v) if isinstance(v, dict) else v) for k, v in ws.__dict__.items()})
        stale, _ = lookback_call(poisoned, 3, 1, random.Random(seed + 1), resident=3, spin_limit=10_000,
                                 stall=(1, 60))
        if stale:
            found = True
            clean = Region()                              # the caller's zero-fill after a timeout
            stale, timed_out = lookback_call(clean, 3, 1, random.Random(seed + 1), resident=3, spin_limit=10_000,
                                             stall=(1, 60))
            assert not timed_out
            assert not stale
    assert found, "the model no longer shows the post-timeout hazard: update the header and this test"
