"""Pins for the LFU slot-cache simulator: hand-traced sequences and invariants."""
import numpy as np

from oracle.lfu_sim import LFUSim


def test_hand_traced_eviction_sequence():
    # 4 slots, steps of 2 ids; traced by hand:
    #  step0 [1,2]: 1 -> slot0 (t1), 2 -> slot1 (t2)               counts s0=1 s1=1
    #  step1 [3,1]: hit 1 (s0 count 2, t3); 3 -> empty slot2 (t4)
    #  step2 [4,5]: 4 -> empty slot3 (t5); 5: victims s0(2,t3) s1(1,t2) s2(1,t4)
    #               -> slot1 (count 1, oldest), t6
    #  step3 [2,3]: hit 3 (s2, t7); 2: victims s0(2,t3) s1(1,t6) s3(1,t5) -> slot3, t8
    sim = LFUSim(1, 4)
    for ids in ([1, 2], [3, 1], [4, 5], [2, 3]):
        sim.step(0, ids)
    assert sim.log == [
        (0, 0, 1, 0, 0), (0, 0, 2, 0, 1),
        (0, 1, 1, 1, 0), (0, 1, 3, 0, 2),
        (0, 2, 4, 0, 3), (0, 2, 5, 0, 1),
        (0, 3, 3, 1, 2), (0, 3, 2, 0, 3),
    ]


def test_hits_before_misses_within_a_step():
    sim = LFUSim(1, 2)
    sim.step(0, [7, 8])
    # 9 misses; 7 hits; the hit is logged first although 9 comes first in the step
    sim.step(0, [9, 7])
    assert sim.log[2:] == [(0, 1, 7, 1, 0), (0, 1, 9, 0, 1)]


def test_compulsory_misses_only_when_ids_fit():
    rng = np.random.default_rng(0)
    sim = LFUSim(2, 16)
    seen = [set(), set()]
    for _ in range(200):
        for layer in (0, 1):
            ids = rng.choice(16, 8, replace=False)
            sim.step(layer, ids)
            seen[layer] |= set(int(e) for e in ids)
    for layer in (0, 1):
        misses = sum(1 for r in sim.log if r[0] == layer and r[3] == 0)
        assert misses == len(seen[layer])


def test_accounting_and_no_self_eviction():
    rng = np.random.default_rng(1)
    sim = LFUSim(3, 16)
    n_acc = 0
    for _ in range(300):
        layer = int(rng.integers(3))
        ids = rng.choice(128, 8, replace=False)
        where = sim.step(layer, ids)
        n_acc += 8
        assert len(set(where.values())) == 8           # distinct slots in one step
        for e, s in where.items():
            assert sim.expert[layer][s] == e           # every id of the step is resident after it
    assert len(sim.log) == n_acc
    hits = sum(r[3] for r in sim.log)
    assert hits + sum(1 - r[3] for r in sim.log) == n_acc
    for layer in range(3):                               # per-layer step counters
        st = [r[1] for r in sim.log if r[0] == layer]
        assert st == sorted(st) and (not st or st[0] == 0)


def test_chunk_steps_resident_first():
    sim = LFUSim(1, 4)
    sim.step(0, [3, 9])
    assert sim.chunk_steps(0, [1, 9, 3, 12, 5, 9], 2) == [[3, 9], [1, 5], [12]]


def test_hand_traced_prefetch():
    # 2 slots, one id per step; traced by hand:
    #  [1] -> s0 (c1, t1); [2] -> s1 (c1, t2); [1] hit s0 (c2, t3);
    #  [3]: victims s0 (2, t3), s1 (1, t2) -> s1 (c1, t4);
    #  [2]: victims s0 (2, t3), s1 (1, t4) -> s1 (c1, t5);
    #  [3]: -> s1 (c1, t6).  Access totals: 1: 2, 2: 2, 3: 2.
    #  prefetch(1): candidates (not resident) [2]; victim s1 (count 1 < 2)
    #               -> 2 into s1 with count 0 (t7), step 6;
    #  prefetch(1): candidates [3]; victim s1 (count 0 < 2) -> 3 into s1 (t8), step 7;
    #  [2]: a miss again: victims s0 (2, t3), s1 (0, t8) -> s1 (t9), step 8.
    sim = LFUSim(1, 2)
    for ids in ([1], [2], [1], [3], [2], [3]):
        sim.step(0, ids)
    assert sim.prefetch(0, 1) == [(2, 1)]
    assert sim.prefetch(0, 1) == [(3, 1)]
    sim.step(0, [2])
    assert sim.log[6:] == [(0, 6, 2, 2, 1), (0, 7, 3, 2, 1), (0, 8, 2, 0, 1)]


def test_prefetch_keeps_hotter_residents():
    # 1 slot: expert 2 resident with count 3; expert 1 accessed once: its
    # victim (count 3) is not colder, so nothing is staged (the step still counts)
    sim = LFUSim(1, 1)
    for ids in ([1], [2], [2], [2]):
        sim.step(0, ids)
    assert sim.prefetch(0, 1) == []
    assert sim.steps[0] == 5 and len(sim.log) == 4
    assert sim.prefetch(0, 0) == [] and sim.steps[0] == 5     # P = 0: no step
