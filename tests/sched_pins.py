"""Pins for the scheduler oracle (coverage, ordering, quota, hand-worked example).

Each ``pin_*`` takes the scheduler module (normally ``oracle.sched_ref``) and
raises AssertionError on disagreement; the mutant tests reuse them.
"""

from __future__ import annotations

import json
import os
import random

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _ceil_div(a, b):
    return -(-a // b)


def check_schedule(sched, seqlens, num_parts, F=5):
    """Invariants any valid output must satisfy (independent of how it was computed)."""
    meta, num_splits = sched.tile_schedule_ref(seqlens, num_parts, F)
    b = len(seqlens)
    n = [_ceil_div(L, 64) for L in seqlens]
    assert len(meta) == num_parts and all(len(m) == 8 for m in meta)
    assert len(num_splits) == b + 1 and num_splits[0] == 0
    assert all(num_splits[i] <= num_splits[i + 1] for i in range(b)), "num_splits not monotone"
    covered = {}
    split_seen = {r: [] for r in range(b)}
    total = sum(x + F for x in n if x > 0)
    share = _ceil_div(total, num_parts) if total else 0
    prev_end = (0, 0)
    for p, m in enumerate(meta):
        if p == 0:
            first = next((r for r in range(b) if n[r] > 0), b)
            assert (m[0], m[1]) == (first, 0), f"part 0 begins at {(m[0], m[1])}"
        else:
            assert (m[0], m[1]) == prev_end, f"part {p} does not start where part {p - 1} ended"
        assert (m[0], m[1]) <= (m[2], m[3]), f"part {p} ends before it begins"
        prev_end = (m[2], m[3])
        chunks = sched.chunks_of_part(m, seqlens)
        load = 0
        for (r, lo, hi, si) in chunks:
            assert 0 <= lo < hi <= n[r]
            for k in range(lo, hi):
                assert (r, k) not in covered, f"block {(r, k)} covered twice"
                covered[(r, k)] = p
            split_seen[r].append(si)
            load += (hi - lo) + F
        if total:
            assert load <= share + F, f"part {p} load {load} above share + F = {share + F}"
            if (p + 1) * share <= total:
                assert load >= share - F, f"part {p} load {load} below share - F = {share - F}"
    assert prev_end == (b, 0), f"partitions do not end at (b, 0): {prev_end}"
    for r in range(b):
        for k in range(n[r]):
            assert (r, k) in covered, f"block {(r, k)} not covered"
        c = num_splits[r + 1] - num_splits[r]
        assert c == len(split_seen[r]), f"request {r}: num_splits says {c}, saw {len(split_seen[r])}"
        assert sorted(split_seen[r]) == list(range(c)), f"request {r}: split indices {split_seen[r]}"
        assert (c == 0) == (n[r] == 0)
    return meta, num_splits


def pin_sched_golden(sched):
    with open(os.path.join(GOLDEN, "sched_small.json")) as f:
        g = json.load(f)
    meta, ns = sched.tile_schedule_ref(g["seqlens"], g["num_parts"], g["fixed_overhead"])
    assert meta == g["expected_meta"], meta
    assert ns == g["expected_num_splits"], ns


def pin_sched_invariants_edges(sched):
    edge = [0, 1, 63, 64, 65, 127, 128, 129, 16384, 4096, 2]
    for P in (1, 2, 3, 37, 74, 148):
        check_schedule(sched, edge, P)
        check_schedule(sched, [0, 0, 0], P)
        check_schedule(sched, [1], P)
        check_schedule(sched, [16384] * 3, P)


def pin_sched_invariants_random(sched):
    rng = random.Random(1234)
    for trial in range(60):
        b = rng.choice([1, 2, 5, 16, 64, 132, 200])
        lens = [rng.choice([0, 1, 63, 64, 65, rng.randint(1, 16384), rng.randint(1, 40000)]) for _ in range(b)]
        P = rng.choice([1, 7, 37, 74, 148])
        check_schedule(sched, lens, P)


def pin_sched_balance(sched):
    """Equal requests: every partition's work (blocks + F per chunk) is within F of the share."""
    lens = [4096] * 128
    P = 74
    meta, _ = sched.tile_schedule_ref(lens, P, 5)
    share = _ceil_div(128 * (64 + 5), P)
    loads = [sum(hi - lo + 5 for (_, lo, hi, _) in sched.chunks_of_part(meta[p], lens)) for p in range(P)]
    assert all(share - 5 <= x <= share + 5 for x in loads[:-1]), loads
    assert sum(x - 5 * len(sched.chunks_of_part(meta[p], lens)) for p, x in enumerate(loads)) == 128 * 64


ALL_SCHED_PINS = [pin_sched_golden, pin_sched_invariants_edges, pin_sched_invariants_random, pin_sched_balance]
