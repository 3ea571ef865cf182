"""Failure detection on the GPU: the per-problem status bits and the bounded
waits, exercised without faulting, trapping or hanging the device.

* NONFINITE / NOT_PD: NaN injected on the host into one problem's inputs.
  The status bits match the oracle's reading of the same inputs, the bad
  problem keeps its previous values, and the other problems of the batch are
  untouched (a whole solve with one poisoned problem leaves every other
  problem bit-identical to a clean run).
* TIMEOUT: kvs_set_wait_limit makes every pipeline wait of the tensor-core
  kernels give up after a few cycles, far too short for any copy to land.
  The kernels then unwind (the waits of the unwinding keep their normal
  limit), the calls with a status array report KVS_ST_TIMEOUT, the calls
  without one return NaN outputs, and after the limit is restored the next
  calls on the same workspace give the same results as before.
"""
import numpy as np
import pytest
import torch

import oracle as O
import workload as W
from gpu_common import Case, dev, host, rel
from test_gpu_parity import SMALL64, run_compress, select_fit_point

pytestmark = pytest.mark.gpu

ST_TIMEOUT = 8


def small():
    return Case(SMALL64, k=[50, 7, 33, 20])


def test_fit_flags_nonfinite_and_not_pd_per_problem():
    c = small()
    K = c.K
    Kcs, _, tgt = select_fit_point(c, 0.2)
    Ys = [t[0].copy() for t in tgt]
    Ys[1][3, 5] = np.nan                       # problem 1: NaN target row
    Qs = [q.copy() for q in c.Qs]
    Qs[2][0, 0] = np.nan                       # problem 2: NaN query
    sentinel = np.full((c.batch.sum_c, c.wl.d), 3.0, np.float32)
    Vc = dev(sentinel)
    status = torch.zeros(c.bt.B, dtype=torch.int32, device="cuda")
    K.kvs_fit_values(c.batch, dev(np.concatenate(Qs)), dev(np.concatenate(Kcs)),
                     dev(np.concatenate(Ys)), 1e-3, Vc, status, c.ws)
    torch.cuda.synchronize()
    st, gv = host(status), host(Vc)
    co = c.batch.c_off_h
    for b in range(c.bt.B):
        Vo, so = O.ridge_fit(Qs[b], Kcs[b], Ys[b], 1e-3)
        assert st[b] == so, (b, st[b], so)
        if so:
            np.testing.assert_array_equal(gv[co[b]:co[b + 1]], sentinel[co[b]:co[b + 1]])
        else:
            assert rel(gv[co[b]:co[b + 1]], Vo) < 1e-3
    assert st[1] == K.ST_NONFINITE and st[2] == K.ST_NOT_PD and st[0] == 0 and st[3] == 0


@pytest.mark.parametrize("where", ["Y", "Q"])
def test_lbfgs_step_flags_a_nonfinite_loss(where):
    c = Case(W.WORKLOADS["single_d64"])
    K = c.K
    Kcs, Vcs, tgt = select_fit_point(c)
    Y = tgt[0][0].copy()
    Q = c.Qs[0].copy()
    if where == "Y":
        Y[4, 2] = np.nan
    else:
        Q[7, 1] = np.nan
    sched = K.Schedule(max_bt=3)
    Kc = dev(Kcs[0])
    state = K.alloc_state(c.batch, sched.history)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    K.kvs_lbfgs_reset(c.batch, sched, dev(Q), dev(Y), dev(tgt[0][1]), dev(Vcs[0]), Kc, state, 1,
                      c.ws)
    K.kvs_lbfgs_step(c.batch, sched, dev(Q), dev(Y), dev(tgt[0][1]), dev(Vcs[0]), Kc, state,
                     status, None, c.ws)
    torch.cuda.synchronize()
    st = int(host(status)[0])
    assert st & K.ST_NONFINITE and st & K.ST_LS_FAIL, st
    np.testing.assert_array_equal(host(Kc), Kcs[0])
    # the oracle reads the same inputs the same way
    d = c.wl.d
    f, g, _ = O.loss_grad(Q, Kcs[0], Vcs[0], Y, tgt[0][1])
    ost = O.LBFGSState(x=Kcs[0].astype(np.float64).ravel(), f=f, g=g.ravel())
    O.lbfgs_step(ost, lambda x: O.loss_only(Q, x.reshape(-1, d), Vcs[0], Y, tgt[0][1]),
                 lambda x: O.loss_grad(Q, x.reshape(-1, d), Vcs[0], Y, tgt[0][1])[1].ravel(),
                 max_bt=3)
    assert ost.status == O.ST_NONFINITE | O.ST_LS_FAIL


def test_solve_isolates_a_poisoned_problem():
    wl = SMALL64.with_(outer=2, steps=3)
    sched_args = dict(outer=wl.outer, steps=wl.steps)
    clean = Case(wl, k=[50, 7, 33, 20])
    bad = Case(wl, k=[50, 7, 33, 20])
    Vz = host(bad.Vz)
    z0 = bad.bt.z_off[2]
    Vz[z0 + 11, 3] = np.nan                   # problem 2's zone values
    bad.Vz = dev(Vz)
    rc = run_compress(clean, clean.K.Schedule(**sched_args))
    rb = run_compress(bad, bad.K.Schedule(**sched_args))
    assert not rc["status"].any()
    assert rb["status"][2] & bad.K.ST_NONFINITE, rb["status"]
    co = clean.batch.c_off_h
    for b in (0, 1, 3):
        assert rb["status"][b] == 0
        np.testing.assert_array_equal(rb["Kc"][co[b]:co[b + 1]], rc["Kc"][co[b]:co[b + 1]])
        np.testing.assert_array_equal(rb["Vc"][co[b]:co[b + 1]], rc["Vc"][co[b]:co[b + 1]])
        np.testing.assert_array_equal(rb["trace"][b], rc["trace"][b])
    # the oracle flags the same problem
    res = O.compress(bad.Qs[2], bad.Zk[2], Vz[z0:bad.bt.z_off[3]], 33,
                     O.Schedule(**sched_args))
    assert res["status"] & O.ST_NONFINITE


def test_wait_timeout_is_reported_and_recovers():
    c = small()
    K = c.K
    Kcs, Vcs, tgt = select_fit_point(c, 0.1)
    args = (c.Q, dev(np.concatenate(Kcs)), dev(np.concatenate(Vcs)),
            dev(np.concatenate([t[0] for t in tgt])), dev(np.concatenate([t[1] for t in tgt])))
    B = c.bt.B

    def loss_grad():
        loss = torch.empty(B, device="cuda")
        parts = torch.empty((B, 2), device="cuda")
        dK = torch.empty((c.batch.sum_c, c.wl.d), device="cuda")
        K.kvs_loss_grad(c.batch, *args, 1.0, 1.0, loss, parts, dK, c.ws)
        torch.cuda.synchronize()
        return host(loss), host(parts), host(dK)

    def fit():
        Vc = torch.zeros((c.batch.sum_c, c.wl.d), device="cuda")
        status = torch.zeros(B, dtype=torch.int32, device="cuda")
        K.kvs_fit_values(c.batch, c.Q, args[1], args[3], 1e-3, Vc, status, c.ws)
        torch.cuda.synchronize()
        return host(Vc), host(status)

    ref = loss_grad()
    ref_fit = fit()
    assert np.isfinite(ref[0]).all() and not ref_fit[1].any()
    try:
        K.kvs_set_wait_limit(16)  # far below the latency of any copy
        lg = loss_grad()
        fv, fst = fit()
        Y = torch.empty_like(c.Q)
        lse = torch.empty(c.Q.shape[0], device="cuda")
        K.kvs_targets(c.batch, c.Q, c.Kz, c.Vz, Y, lse, None, c.ws)
        torch.cuda.synchronize()
    finally:
        K.kvs_set_wait_limit(0)
    assert all(np.isnan(x).all() for x in lg), "loss_grad outputs must all be NaN"
    assert np.isnan(host(Y)).all() and np.isnan(host(lse)).all()
    assert np.all(fst & ST_TIMEOUT), fst
    # the device and the workspace are still good: the same results as before
    again = loss_grad()
    for a, b in zip(again, ref):
        np.testing.assert_array_equal(a, b)
    v2, s2 = fit()
    assert not s2.any()
    np.testing.assert_array_equal(v2, ref_fit[0])
    with pytest.raises(K.KvsError):
        K.kvs_set_wait_limit(-1)
