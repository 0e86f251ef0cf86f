"""The C++ LFU planner (libmoe, planning-only handle, no GPU) against the
reference simulator, access by access."""
import numpy as np
import pytest

from oracle.lfu_sim import LFUSim


@pytest.fixture(scope="module")
def M():
    import quantized_moe_bit_b200 as M
    return M


def test_hand_traced_sequence(M):
    lf = M.MoeLfu(1, 16, 4)
    for ids in ([1, 2], [3, 1], [4, 5], [2, 3]):
        lf.plan(0, ids)
    assert lf.log() == [
        (0, 0, 1, 0, 0), (0, 0, 2, 0, 1),
        (0, 1, 1, 1, 0), (0, 1, 3, 0, 2),
        (0, 2, 4, 0, 3), (0, 2, 5, 0, 1),
        (0, 3, 3, 1, 2), (0, 3, 2, 0, 3),
    ]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_random_streams_match_simulator(M, seed):
    rng = np.random.default_rng(seed)
    L, E, S, k = 3, 128, 16, 8
    lf = M.MoeLfu(L, E, S)
    sim = LFUSim(L, S)
    p = np.arange(1, E + 1, dtype=np.float64) ** -1.1
    p /= p.sum()
    for it in range(400):
        layer = int(rng.integers(L))
        if rng.random() < 0.2:
            # a prefill chunk: distinct experts cut into steps, resident first
            distinct = sorted(set(rng.choice(E, 60, p=p).tolist()))
            for ids in sim.chunk_steps(layer, distinct, k):
                slots, hits = lf.plan(layer, ids)
                where = sim.step(layer, ids)
                assert slots == [where[e] for e in ids]
        else:
            ids = [int(e) for e in rng.choice(E, k, replace=False, p=p)]
            slots, hits = lf.plan(layer, ids)
            where = sim.step(layer, ids)
            assert slots == [where[e] for e in ids]
        if rng.random() < 0.25:
            # a lookahead prefetch of up to P experts of the layer
            P = int(rng.integers(1, 4))
            ids, slots = lf.plan_prefetch(layer, P)
            assert list(zip(ids, slots)) == sim.prefetch(layer, P)
    assert lf.log() == sim.log
    assert any(r[3] == 2 for r in sim.log)
    h, m, _ = lf.stats()
    assert h == sum(1 for r in sim.log if r[3] == 1) and m == sum(1 for r in sim.log if r[3] == 0)


def test_invalid_steps(M):
    lf = M.MoeLfu(2, 16, 4)
    with pytest.raises(M.MoeError):
        lf.plan(0, [1, 1])                 # repeated id
    with pytest.raises(M.MoeError):
        lf.plan(0, [1, 99])                # out of range
    with pytest.raises(M.MoeError):
        lf.plan(0, [0, 1, 2, 3, 4])        # more ids than slots
    with pytest.raises(M.MoeError):
        lf.plan(2, [0])                    # layer out of range
    assert lf.log() == []
