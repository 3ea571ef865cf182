"""Random-restart search (CPU): the seeded restart draws, the replicated batch
layout and the importance mask that selects a chosen subset, and the oracle's
restart search (summary §4 "Optimizer Efficacy" compares a single run with the
best of many restarts)."""
import numpy as np
import pytest

import oracle as O
import workload as W
from kv_cache_compression_kvsculpt_b200 import restarts as RS


def test_restart_inits_are_seeded_distinct_sorted_subsets():
    z, k = [30, 7, 50], [5, 7, 1]
    a = W.restart_inits(z, k, 4, seed=3)
    b = W.restart_inits(z, k, 4, seed=3)
    assert a.shape == (4, 13) and a.dtype == np.int32
    assert np.array_equal(a, b)                       # reproducible
    assert not np.array_equal(a, W.restart_inits(z, k, 4, seed=4))
    off = np.concatenate([[0], np.cumsum(k)])
    for r in range(4):
        for i in range(3):
            s = a[r, off[i]:off[i + 1]]
            assert np.all(np.diff(s) > 0) and s.min() >= 0 and s.max() < z[i]
    assert np.array_equal(a[:, 5:12], np.tile(np.arange(7), (4, 1)))  # k = z: the whole zone
    assert len({tuple(a[r, :5]) for r in range(4)}) > 1               # restarts differ
    with pytest.raises(ValueError):
        W.restart_inits([3], [4], 1)


def test_replicate_offsets():
    np.testing.assert_array_equal(RS.replicate_offsets([0, 5, 12], 3),
                                  [0, 5, 12, 17, 24, 29, 36])
    np.testing.assert_array_equal(RS.replicate_offsets([0, 4], 1), [0, 4])


def test_init_mask_selects_exactly_the_chosen_keys():
    z_off = np.array([0, 6, 10])
    c_off = np.array([0, 2, 5])
    inits = np.array([[5, 0, 1, 2, 3], [1, 4, 3, 0, 2]])
    m = RS.init_mask(z_off, c_off, inits)
    assert m.shape == (20,)
    # the oracle's top-k on this mask (ties to the lower position) returns the choice
    for r in range(2):
        for b in range(2):
            zb = m[r * 10 + z_off[b]:r * 10 + z_off[b + 1]]
            kb = c_off[b + 1] - c_off[b]
            assert np.array_equal(O.topk_select(zb.astype(np.float64), kb),
                                  np.sort(inits[r, c_off[b]:c_off[b + 1]]))
    with pytest.raises(ValueError):
        RS.init_mask(z_off, c_off, np.array([[1, 1, 0, 1, 2]]))   # repeated position
    with pytest.raises(ValueError):
        RS.init_mask(z_off, c_off, np.array([[0, 6, 0, 1, 2]]))   # outside the zone


def test_oracle_restart_search():
    r = np.random.default_rng(31)
    Q = r.standard_normal((24, 4))
    Kz = r.standard_normal((10, 4))
    Vz = r.standard_normal((10, 4))
    sched = O.Schedule(outer=2, steps=3)
    single = O.compress(Q, Kz, Vz, 3, sched)
    # a restart from the top-k keys is the single run
    runs, best = O.restart_search(Q, Kz, Vz, 3, sched, [single["idx"]])
    assert best == 0 and runs[0]["loss"] == single["loss"]
    np.testing.assert_array_equal(runs[0]["trace"], single["trace"])
    inits = W.restart_inits([10], [3], 5, seed=1)
    runs, best = O.restart_search(Q, Kz, Vz, 3, sched, inits)
    losses = [x["loss"] for x in runs]
    assert best == int(np.argmin(losses))
    for x, ix in zip(runs, inits):
        assert np.array_equal(x["idx"], ix)           # each run starts from its subset
        assert np.all(np.diff(x["trace"]) <= 1e-15)   # and never raises its loss
