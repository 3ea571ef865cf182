"""Pins of the oracle's alternating schedule and of its adaptive driver.

"KVSculpt: KV Cache Compression as Distillation": the abstract has keys
optimised by L-BFGS and values re-solved in closed form, alternating every few
steps; summary section 2 "Optimization Strategy" and "Value Optimization"
describe the two halves and "Adaptive Budget Allocation" the pilot run that
sets each problem's budget.  These tests tie `oracle.compress` and
`oracle.adaptive_compress` to facts that hold whatever the trajectory is:

* after every value fit the reported loss is the loss evaluated from scratch
  at that fit's (K_c, V_c), and V_c is the ridge solution at those keys (a
  stale loss or gradient carried over from before the fit fails this);
* the keys entering fit o are the result of `steps` L-BFGS steps, each of
  which meets the Armijo condition against a fresh evaluation;
* the history flag: clearing the (s, y) pairs at every fit and keeping them
  are different runs, and each equals a run whose pairs are kept or cleared by
  hand around the oracle's own L-BFGS step;
* zero L-BFGS steps reduce the schedule to Select+Fit;
* the adaptive driver spends exactly the budget, allocates by the pilot's
  output MSE (never less budget to a problem with a larger pilot MSE), and runs
  each full solve at its allocated size with the full schedule.
CPU only.
"""
import numpy as np
import pytest

import oracle as O


def problem(n_q=40, z=20, d=8, seed=0, key_scale=1.0):
    r = np.random.default_rng(seed)
    Q = r.standard_normal((n_q, d))
    Kz = r.standard_normal((z, d)) * key_scale
    Vz = r.standard_normal((z, d))
    return Q, Kz, Vz


@pytest.mark.parametrize("persist", [True, False])
def test_trace_is_a_fresh_loss_after_every_fit(persist):
    Q, Kz, Vz = problem(seed=3)
    k = 6
    sched = O.Schedule(outer=5, steps=3, persist_history=persist)
    rec = []
    r = O.compress(Q, Kz, Vz, k, sched, record=rec)
    Y, lse = O.targets(Q, Kz, Vz)
    assert len(rec) == sched.outer + 1 == len(r["trace"])
    idx = O.topk_select(O.importance(Q, Kz, lse), k)
    np.testing.assert_array_equal(rec[0][0], Kz[idx])
    for o, (Kc, Vc, _) in enumerate(rec):
        # V_c is the ridge solution at the fit's keys: the normal equations hold
        A, _ = O.attention(Q, Kc)
        G = A.T @ A + sched.lam * np.eye(k)
        res = G @ Vc - A.T @ Y
        assert np.linalg.norm(res) <= 1e-10 * np.linalg.norm(A.T @ Y)
        # the reported loss is the loss at (K_c, V_c), evaluated from scratch
        f = O.loss_only(Q, Kc, Vc, Y, lse)
        assert abs(r["trace"][o] - f) <= 1e-13 * max(f, 1e-300), o
    # the final result is the last fit's state
    np.testing.assert_array_equal(r["Kc"], rec[-1][0])
    np.testing.assert_array_equal(r["Vc"], rec[-1][1])
    assert r["loss"] == pytest.approx(r["trace"][-1], rel=1e-14)


def test_keys_between_fits_come_from_armijo_steps_at_fixed_values():
    """Replaying one outer iteration: the keys of fit o+1 are reached from those
    of fit o by `steps` L-BFGS steps at the values of fit o, each accepted step
    meeting the Armijo condition against a fresh loss."""
    Q, Kz, Vz = problem(seed=5)
    k, d = 5, 8
    sched = O.Schedule(outer=3, steps=4, persist_history=False)
    rec = []
    O.compress(Q, Kz, Vz, k, sched, record=rec)
    Y, lse = O.targets(Q, Kz, Vz)
    for o in range(sched.outer):
        Kc, Vc, _ = rec[o]
        f, g, _ = O.loss_grad(Q, Kc, Vc, Y, lse)
        st = O.LBFGSState(x=Kc.ravel().copy(), f=f, g=g.ravel())
        for _ in range(sched.steps):
            x0, f0 = st.x.copy(), st.f
            ok = O.lbfgs_step(st, lambda x: O.loss_only(Q, x.reshape(-1, d), Vc, Y, lse),
                              lambda x: O.loss_grad(Q, x.reshape(-1, d), Vc, Y, lse)[1].ravel())
            if ok:
                assert O.loss_only(Q, st.x.reshape(-1, d), Vc, Y, lse) <= f0
                assert st.f == pytest.approx(O.loss_only(Q, st.x.reshape(-1, d), Vc, Y, lse),
                                             rel=1e-13)
            else:
                np.testing.assert_array_equal(st.x, x0)
        np.testing.assert_allclose(st.x.reshape(-1, d), rec[o + 1][0], rtol=0, atol=1e-12)


def manual_schedule(Q, Kz, Vz, k, sched, keep_pairs):
    """The schedule written out around the oracle's own steps, with the pairs
    kept or cleared by hand at every fit."""
    d = Q.shape[1]
    Y, lse = O.targets(Q, Kz, Vz)
    Kc = Kz[O.topk_select(O.importance(Q, Kz, lse), k)]
    Vc, _ = O.ridge_fit(Q, Kc, Y, sched.lam)
    f, g, _ = O.loss_grad(Q, Kc, Vc, Y, lse)
    st = O.LBFGSState(x=Kc.ravel().copy(), f=f, g=g.ravel())
    trace = [f]
    for _o in range(sched.outer):
        for _t in range(sched.steps):
            O.lbfgs_step(st, lambda x: O.loss_only(Q, x.reshape(-1, d), Vc, Y, lse),
                         lambda x: O.loss_grad(Q, x.reshape(-1, d), Vc, Y, lse)[1].ravel(),
                         sched.history)
        Vc, _ = O.ridge_fit(Q, st.x.reshape(-1, d), Y, sched.lam)
        if not keep_pairs:
            st.hist_s, st.hist_y = [], []
        f, g, _ = O.loss_grad(Q, st.x.reshape(-1, d), Vc, Y, lse)
        st.f, st.g = f, g.ravel()
        trace.append(f)
    return np.array(trace)


def test_history_flag_keeps_or_clears_the_pairs():
    Q, Kz, Vz = problem(n_q=48, z=24, seed=11, key_scale=1.5)
    k = 6
    runs = {}
    for persist in (True, False):
        sched = O.Schedule(outer=4, steps=4, persist_history=persist)
        rec = []
        r = O.compress(Q, Kz, Vz, k, sched, record=rec)
        runs[persist] = r["trace"]
        np.testing.assert_allclose(r["trace"], manual_schedule(Q, Kz, Vz, k, sched, persist),
                                   rtol=1e-12, atol=0)
        pairs = [c for _, _, c in rec[1:]]
        if persist:
            # pairs survive the fits: the count grows past one block's steps
            assert max(pairs) > sched.steps
        else:
            assert all(c == 0 for c in pairs)
    # the two settings give different trajectories on this problem
    assert np.max(np.abs(runs[True][2:] - runs[False][2:])) > 1e-9 * runs[True][0]


def test_zero_steps_is_select_fit():
    Q, Kz, Vz = problem(seed=7)
    k = 5
    r = O.compress(Q, Kz, Vz, k, O.Schedule(outer=2, steps=0))
    Y, lse = O.targets(Q, Kz, Vz)
    idx = O.topk_select(O.importance(Q, Kz, lse), k)
    V0, _ = O.ridge_fit(Q, Kz[idx], Y, 1e-3)
    sf = O.loss_only(Q, Kz[idx], V0, Y, lse)
    np.testing.assert_allclose(r["trace"], [sf, sf, sf], rtol=1e-14)
    np.testing.assert_array_equal(r["Kc"], Kz[idx])
    assert r["trials"] == 0


def test_adaptive_driver_follows_the_pilot():
    # four problems of graded difficulty: the key scale sharpens attention
    probs = [dict(zip(("Q", "Kz", "Vz"), problem(n_q=40, z=24, seed=20 + i, key_scale=s)))
             for i, s in enumerate((0.5, 1.0, 2.0, 3.0))]
    total, k_min = 4 * 8, 3
    sched = O.Schedule(outer=3, steps=3)
    pilot = O.Schedule(outer=1, steps=2)
    res = O.adaptive_compress(probs, total, sched, pilot, k_min=k_min, alpha=0.5)
    k = res["k"]
    assert int(k.sum()) == total and np.all(k >= k_min)
    assert np.all(k <= [len(p["Kz"]) for p in probs])
    # the pilot ran at the uniform size with the pilot schedule: its signal is the
    # output-MSE term after the pilot's last fit
    for p, m in zip(probs, res["pilot_mse"]):
        rp = O.compress(p["Q"], p["Kz"], p["Vz"], total // len(probs), pilot)
        assert len(rp["trace"]) == pilot.outer + 1
        assert m == pytest.approx(rp["mse_out"], rel=1e-12)
    # more pilot error never receives less budget
    order = np.argsort(res["pilot_mse"])
    assert np.all(np.diff(k[order]) >= 0)
    assert len(set(k.tolist())) > 1, "the pilot signal should separate these problems"
    # each full solve runs at its allocated size with the full schedule
    for p, kb, r in zip(probs, k, res["results"]):
        assert r["Kc"].shape == (kb, p["Q"].shape[1])
        assert len(r["trace"]) == sched.outer + 1
        want = O.compress(p["Q"], p["Kz"], p["Vz"], int(kb), sched)
        assert r["loss"] == pytest.approx(want["loss"], rel=1e-12)
