"""The softmax turn protocol of the two-tile attention kernel, as a host-side
model (no GPU). Within a unit the softmax warpgroups of query tiles 0 and 1
hand the exponential turn to each other through two mbarriers (turn[0]
awaited by tile 0, turn[1] by tile 1), and each waits with a phase-parity
wait. A parity wait cannot tell phase p from phase p + 2, so an arrival must
never complete a barrier's next phase before its waiter has consumed the
previous one.

The rules below restate the kernel's: which step waits, which step hands
over, and the hand-back at the end of a unit that tile 0 ends by handing over
(`ret`). The test runs both tiles through random unit sequences in random
interleavings, with no other ordering between them (the kernel's S, P, Q and
K/V barriers only remove interleavings). It checks that no arrival lands on
a barrier whose previous phase is unconsumed, and that every sequence runs to
its end. Without the hand-back (the e4m3 kernels' rules) the same search finds
interleavings that break this. There, the loader's order forbids them:
tile 0 cannot begin a unit before tile 1 has issued its last Q K^T of the
previous one.
"""

from __future__ import annotations

import random

import pytest


def _ops(units, t, ranges, hand_back):
    """The turn operations of tile t over a CTA's units: ('wait', b) or ('arrive', b)."""
    ops = []
    turn_back = False
    for n0, n1 in units:
        ret = hand_back and n0 >= 1 and n0 <= n1
        n = n1 if t else n0
        for j in range(n):
            if ranges:
                wait = (j >= 1 and j - 1 < n1) if t == 0 else j < n0
                hand = (j < n1) if t == 0 else j + 1 < n0
            else:
                wait = j >= 1 if t == 0 else j < n0
                hand = (t == 0) or j + 1 < n0
            if hand_back and t == 0 and j == 0:
                wait = turn_back
                turn_back = False
            if hand_back and t == 1 and ret and j == n0 - 1:
                hand = True
            if wait:
                ops.append(("wait", t))
            if hand:
                ops.append(("arrive", 1 - t))
        if hand_back and t == 0 and ret:
            turn_back = True
    return ops


def _run(units, ranges, hand_back, rng):
    """Interleave the two tiles at random. Returns 'ok', 'aba' or 'deadlock'."""
    ops = [_ops(units, 0, ranges, hand_back), _ops(units, 1, ranges, hand_back)]
    pos = [0, 0]
    arrived = [0, 0]   # phases completed on turn[b]
    consumed = [0, 0]  # phases its waiter has seen
    while pos[0] < len(ops[0]) or pos[1] < len(ops[1]):
        ready = []
        for t in (0, 1):
            if pos[t] == len(ops[t]):
                continue
            kind, b = ops[t][pos[t]]
            if kind == "arrive" or arrived[b] > consumed[b]:
                ready.append(t)
        if not ready:
            return "deadlock"
        t = rng.choice(ready)
        kind, b = ops[t][pos[t]]
        if kind == "arrive":
            if arrived[b] > consumed[b]:
                return "aba"
            arrived[b] += 1
        else:
            consumed[b] += 1
        pos[t] += 1
    return "ok"


def _units(rng, ranges, count):
    units = []
    for _ in range(count):
        if ranges:  # window / pair split: any split of steps, either tile may be empty
            units.append((rng.randint(0, 5), rng.randint(0, 5)))
        else:       # tile 1 sees at least the keys tile 0 sees; empty key-split ranges
            n0 = rng.choice([0, 0, 1, 2, 3, 6])
            units.append((n0, n0 + rng.choice([0, 0, 1, 3])))
    return units


@pytest.mark.parametrize("ranges", [False, True])
def test_hand_back_keeps_every_interleaving_safe(ranges):
    rng = random.Random(1234 + ranges)
    for _ in range(3000):
        units = _units(rng, ranges, rng.randint(1, 8))
        assert _run(units, ranges, True, rng) == "ok", units


def test_per_unit_counts_pair_up_with_the_hand_back():
    """Per barrier, waits = arrivals except the kernel's last hand-back."""
    rng = random.Random(7)
    for ranges in (False, True):
        for _ in range(500):
            units = _units(rng, ranges, rng.randint(1, 6))
            ops = _ops(units, 0, ranges, True) + _ops(units, 1, ranges, True)
            for b in (0, 1):
                arrivals = sum(1 for k, x in ops if k == "arrive" and x == b)
                waits = sum(1 for k, x in ops if k == "wait" and x == b)
                assert 0 <= arrivals - waits <= 1
            last_ret = [u for u in units if u[0] >= 1]
            expect_left = 1 if last_ret and last_ret[-1][0] <= last_ret[-1][1] else 0
            a0 = sum(1 for k, x in ops if k == "arrive" and x == 0)
            w0 = sum(1 for k, x in ops if k == "wait" and x == 0)
            assert a0 - w0 == expect_left


def test_without_the_hand_back_an_unordered_interleaving_breaks():
    """The e4m3 rules rely on the loader's order: in a free interleaving, tile
    0 can hand over twice (end of one unit, first step of the next) before
    tile 1 has waited once."""
    rng = random.Random(99)
    units = [(2, 2), (2, 2)]
    results = {_run(units, False, False, rng) for _ in range(200)}
    assert "aba" in results
