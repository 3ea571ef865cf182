"""Pins of the float64 oracle against facts that do not come from the oracle.

Each test ties one oracle function to a closed form, an invariant, a brute-force
enumeration, an independent library route or a hand-derived example, so that a
dropped term, a wrong sign or index or a transposed operand fails at least one
of them.  CPU only.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.special

import oracle as O

RNG = np.random.default_rng(1234)


def tiny(n_q=5, z=7, k=3, d=4, seed=0, scale=1.0):
    r = np.random.default_rng(seed)
    Q = r.standard_normal((n_q, d)) * scale
    Kz = r.standard_normal((z, d)) * scale
    Vz = r.standard_normal((z, d))
    Kc = r.standard_normal((k, d)) * scale
    Vc = r.standard_normal((k, d))
    return Q, Kz, Vz, Kc, Vc


# --------------------------------------------------------------------- RoPE

def test_rope_matches_complex_rotation():
    """RoPE as multiplication of (x_i + i x_{i+d/2}) by exp(i p theta_i)."""
    d, base = 8, 1e6
    x = RNG.standard_normal((5, d))
    pos = np.array([0, 1, 17, 255, 8191])
    theta = base ** (-2.0 * np.arange(d // 2) / d)
    z = (x[:, :d // 2] + 1j * x[:, d // 2:]) * np.exp(1j * pos[:, None] * theta[None, :])
    want = np.concatenate([z.real, z.imag], axis=1)
    np.testing.assert_allclose(O.rope(x, pos, base), want, rtol=0, atol=1e-12)


def test_rope_d2_closed_form():
    """d=2: theta_0 = 1, so RoPE([1, 0], p) = [cos p, sin p]."""
    p = np.array([0.0, 1.0, 3.0])
    got = O.rope(np.tile([[1.0, 0.0]], (3, 1)), p, 10000.0)
    np.testing.assert_allclose(got, np.stack([np.cos(p), np.sin(p)], 1), atol=1e-15)


def test_rope_relative_position_and_inverse():
    d, base = 16, 1e6
    q = RNG.standard_normal((1, d))
    k = RNG.standard_normal((1, d))
    dots = [float((O.rope(q, [t], base) @ O.rope(k, [t - 5], base).T)[0, 0])
            for t in (5, 100, 2047, 9000)]
    np.testing.assert_allclose(dots, dots[0], rtol=1e-11)
    x = RNG.standard_normal((4, d))
    pos = np.array([3, 77, 1000, 4096])
    np.testing.assert_allclose(O.derope(O.rope(x, pos, base), pos, base), x, atol=1e-13)
    np.testing.assert_allclose(np.linalg.norm(O.rope(x, pos, base), axis=1),
                               np.linalg.norm(x, axis=1), rtol=1e-13)


def test_build_queries_relative_shift_and_order():
    """A synthetic query at N+j scores a key at N+j-D like its context query scores a key at pos-D."""
    g, m_q, n_syn, N, d, base = 2, 3, 4, 64, 8, 1e4
    q_ret = RNG.standard_normal((g * m_q, d))
    q_ctx = RNG.standard_normal((g * n_syn, d))
    pos = np.sort(RNG.choice(N, (g, n_syn)), axis=1).reshape(-1)
    Q = O.build_queries(q_ret, q_ctx, pos, g, m_q, n_syn, N, base)
    assert Q.shape == (g * (m_q + n_syn), d)
    kk = RNG.standard_normal((1, d))
    for h in range(g):
        row0 = h * (m_q + n_syn)
        np.testing.assert_array_equal(Q[row0:row0 + m_q], q_ret[h * m_q:(h + 1) * m_q])
        for j in range(n_syn):
            qs = Q[row0 + m_q + j]
            qc = q_ctx[h * n_syn + j]
            p = pos[h * n_syn + j]
            for D in (0, 3, 40):
                a = float(qs @ O.rope(kk, [N + j - D], base)[0])
                b = float(qc @ O.rope(kk, [p - D], base)[0])
                assert abs(a - b) < 1e-10 * (1 + abs(b))


# ------------------------------------------------------------- attention

def test_targets_brute_force_loops():
    Q, Kz, Vz, _, _ = tiny(n_q=3, z=4, d=3, seed=3)
    Y, lse = O.targets(Q, Kz, Vz)
    s = 1 / math.sqrt(3)
    for i in range(3):
        w = [math.exp(s * sum(Q[i, t] * Kz[j, t] for t in range(3))) for j in range(4)]
        tot = sum(w)
        assert abs(lse[i] - math.log(tot)) < 1e-13
        for c in range(3):
            assert abs(Y[i, c] - sum(w[j] * Vz[j, c] for j in range(4)) / tot) < 1e-13


def test_attention_matches_scipy_and_large_scores():
    Q, Kz, _, _, _ = tiny(n_q=6, z=9, d=8, seed=4, scale=6.0)  # scores up to ~100: needs the max shift
    A, lse = O.attention(Q, Kz)
    S = Q @ Kz.T / math.sqrt(8)
    np.testing.assert_allclose(lse, scipy.special.logsumexp(S, axis=1), rtol=1e-13)
    np.testing.assert_allclose(A, scipy.special.softmax(S, axis=1), rtol=1e-12, atol=1e-300)
    np.testing.assert_allclose(A.sum(1), 1.0, rtol=1e-13)


def test_lse_merge_identity():
    """Chunk-local (Y, l) over two chunks merge to attention over their union."""
    Q, K1, V1, _, _ = tiny(n_q=4, z=5, d=6, seed=5)
    _, K2, V2, _, _ = tiny(n_q=4, z=3, d=6, seed=6)
    Y1, l1 = O.targets(Q, K1, V1)
    Y2, l2 = O.targets(Q, K2, V2)
    Y, l = O.targets(Q, np.vstack([K1, K2]), np.vstack([V1, V2]))
    lm = np.logaddexp(l1, l2)
    np.testing.assert_allclose(l, lm, rtol=1e-13)
    np.testing.assert_allclose(Y, np.exp(l1 - lm)[:, None] * Y1 + np.exp(l2 - lm)[:, None] * Y2,
                               rtol=1e-12)


def test_importance_column_sums():
    Q, Kz, Vz, _, _ = tiny(n_q=5, z=6, d=4, seed=7)
    _, lse = O.targets(Q, Kz, Vz)
    imp = O.importance(Q, Kz, lse)
    assert abs(imp.sum() - 5.0) < 1e-12  # each query's probabilities sum to one
    S = Q @ Kz.T / 2.0
    for j in range(6):
        want = sum(math.exp(S[i, j]) / sum(math.exp(S[i, t]) for t in range(6)) for i in range(5))
        assert abs(imp[j] - want) < 1e-13


# ------------------------------------------------------------------ top-k

@pytest.mark.parametrize("z,k", [(6, 1), (6, 3), (7, 4), (8, 8)])
def test_topk_brute_force_with_ties(z, k):
    r = np.random.default_rng(z * 10 + k)
    imp = r.integers(0, 3, size=z).astype(np.float64)  # many exact ties
    got = O.topk_select(imp, k)
    winners = []
    for sub in itertools.combinations(range(z), k):
        out = [j for j in range(z) if j not in sub]
        if all(imp[i] > imp[j] or (imp[i] == imp[j] and i < j) for i in sub for j in out):
            winners.append(sub)
    assert len(winners) == 1
    assert tuple(got) == winners[0]
    assert list(got) == sorted(got)


# ------------------------------------------------------------------ ridge

def _ridge_obj(A, V, Y, lam):
    return float(((A @ V - Y) ** 2).sum() + lam * (V ** 2).sum())


def test_ridge_normal_equations_and_lstsq():
    Q, Kz, Vz, Kc, _ = tiny(n_q=40, z=30, k=12, d=8, seed=8)
    Y, _ = O.targets(Q, Kz, Vz)
    lam = 1e-3
    V, st = O.ridge_fit(Q, Kc, Y, lam)
    assert st == O.ST_OK
    A, _ = O.attention(Q, Kc)
    R = A.T @ Y
    res = (A.T @ A + lam * np.eye(12)) @ V - R
    assert np.linalg.norm(res) / np.linalg.norm(R) < 1e-10
    # independent route: least squares of the stacked system [A; sqrt(lam) I] V = [Y; 0]
    M = np.vstack([A, math.sqrt(lam) * np.eye(12)])
    rhs = np.vstack([Y, np.zeros((12, 8))])
    V2 = np.linalg.lstsq(M, rhs, rcond=None)[0]
    np.testing.assert_allclose(V, V2, rtol=1e-7, atol=1e-9)
    base = _ridge_obj(A, V, Y, lam)
    for _ in range(5):
        assert _ridge_obj(A, V + 1e-4 * RNG.standard_normal(V.shape), Y, lam) > base


def test_ridge_k1_closed_form():
    """k = 1: every weight is 1, so V = sum_i Y_i / (n_q + lam)."""
    Q, Kz, Vz, Kc, _ = tiny(n_q=9, z=5, k=1, d=4, seed=9)
    Y, _ = O.targets(Q, Kz, Vz)
    V, _ = O.ridge_fit(Q, Kc, Y, 0.25)
    np.testing.assert_allclose(V[0], Y.sum(0) / (9 + 0.25), rtol=1e-13)


def test_ridge_not_pd_flag():
    """Duplicate keys make A^T A singular; a negative penalty then makes the
    Gram matrix indefinite (eigenvalue lam < 0), so the Cholesky must fail."""
    Q, Kz, Vz, Kc, _ = tiny(n_q=6, z=5, k=2, d=4, seed=10)
    Kc[1] = Kc[0]
    Y, _ = O.targets(Q, Kz, Vz)
    V, st = O.ridge_fit(Q, Kc, Y, -1e-3)
    assert V is None and st & O.ST_NOT_PD


# ------------------------------------------------------------ loss / grad

def test_gradient_central_differences():
    Q, Kz, Vz, Kc, Vc = tiny(n_q=5, z=7, k=3, d=4, seed=11)
    Y, lse = O.targets(Q, Kz, Vz)
    f, g, _ = O.loss_grad(Q, Kc, Vc, Y, lse, 0.7, 1.3)
    assert abs(f - O.loss_only(Q, Kc, Vc, Y, lse, 0.7, 1.3)) < 1e-15
    h = 1e-6
    num = np.zeros_like(Kc)
    for a in range(Kc.shape[0]):
        for b in range(Kc.shape[1]):
            kp, km = Kc.copy(), Kc.copy()
            kp[a, b] += h
            km[a, b] -= h
            num[a, b] = (O.loss_only(Q, kp, Vc, Y, lse, 0.7, 1.3)
                         - O.loss_only(Q, km, Vc, Y, lse, 0.7, 1.3)) / (2 * h)
    assert np.linalg.norm(num - g) / np.linalg.norm(g) < 1e-7


def test_loss_terms_by_hand():
    Q, Kz, Vz, Kc, Vc = tiny(n_q=4, z=5, k=2, d=4, seed=12)
    Y, lse = O.targets(Q, Kz, Vz)
    Yh, lh = O.targets(Q, Kc, Vc)
    f, _, parts = O.loss_grad(Q, Kc, Vc, Y, lse, 2.0, 3.0)
    out = sum((Yh[i, c] - Y[i, c]) ** 2 for i in range(4) for c in range(4)) / 16
    ls = sum((lh[i] - lse[i]) ** 2 for i in range(4)) / 4
    assert abs(parts["out"] - out) < 1e-14 and abs(parts["lse"] - ls) < 1e-14
    assert abs(f - (2 * out + 3 * ls)) < 1e-14


def test_full_budget_identity():
    """k = z with K_c = K_z: V_c = V_z reproduces the zone exactly; the ridge
    fit's loss is O(lambda) and vanishes with it."""
    Q, Kz, Vz, _, _ = tiny(n_q=30, z=6, d=8, seed=13)
    Y, lse = O.targets(Q, Kz, Vz)
    f, g, _ = O.loss_grad(Q, Kz, Vz, Y, lse)
    assert f < 1e-28 and np.abs(g).max() < 1e-14
    losses = []
    for lam in (1e-2, 1e-4, 1e-6):
        V, _ = O.ridge_fit(Q, Kz, Y, lam)
        losses.append(O.loss_only(Q, Kz, V, Y, lse))
    assert losses[0] > losses[1] > losses[2] and losses[2] < 1e-9


def test_permutation_invariance():
    Q, Kz, Vz, Kc, Vc = tiny(n_q=8, z=6, k=4, d=4, seed=14)
    Y, lse = O.targets(Q, Kz, Vz)
    f, g, _ = O.loss_grad(Q, Kc, Vc, Y, lse)
    p = np.array([2, 0, 3, 1])
    f2, g2, _ = O.loss_grad(Q, Kc[p], Vc[p], Y, lse)
    assert abs(f - f2) < 1e-14
    np.testing.assert_allclose(g2, g[p], rtol=1e-12)


# ----------------------------------------------------------------- L-BFGS

def test_two_loop_equals_dense_bfgs_inverse_update():
    n = 7
    hs, hy = [], []
    for i in range(4):
        s = RNG.standard_normal(n)
        y = s + 0.3 * RNG.standard_normal(n)  # keeps s^T y > 0
        hs.append(s)
        hy.append(y)
    g = RNG.standard_normal(n)
    gamma = float(hs[-1] @ hy[-1]) / float(hy[-1] @ hy[-1])
    H = gamma * np.eye(n)
    for s, y in zip(hs, hy):
        rho = 1.0 / float(s @ y)
        E = np.eye(n) - rho * np.outer(s, y)
        H = E @ H @ E.T + rho * np.outer(s, s)
    np.testing.assert_allclose(O.two_loop_direction(g, hs, hy), -H @ g, rtol=1e-11)
    np.testing.assert_allclose(O.two_loop_direction(g, [], []), -g)


@pytest.mark.parametrize("c1", [1e-4, 0.5])
def test_armijo_halving_count_on_quadratic(c1):
    """f(x) = a x^2 / 2, empty history: d = -g, t0 = min(1, 1/|g|), the accepted
    step is t0 / 2^j with j the least integer meeting the Armijo condition.
    With u = t a the condition reads (1-u)^2 <= 1 - 2 c1 u, so c1 = 0.5 rejects
    the steps 1 < u < 2 that plain decrease would take (first case: u = 5/3)."""
    for a, x0 in [(50.0, 0.3), (3.0, 2.0), (400.0, -0.01)]:
        f = lambda x: 0.5 * a * float(x[0]) ** 2
        gr = lambda x: np.array([a * float(x[0])])
        st = O.LBFGSState(x=np.array([x0]), f=f([x0]), g=gr([x0]))
        g0 = a * x0
        t = min(1.0, 1.0 / abs(g0))
        while not (0.5 * a * (x0 - t * g0) ** 2 <= 0.5 * a * x0 ** 2 - c1 * t * g0 * g0):
            t *= 0.5
        assert O.lbfgs_step(st, f, gr, c1=c1)
        assert abs(st.x[0] - (x0 - t * g0)) < 1e-15


def test_lbfgs_solves_convex_quadratic():
    n = 12
    M = RNG.standard_normal((n, n))
    H = M @ M.T + 0.5 * np.eye(n)
    b = RNG.standard_normal(n)
    xs = np.linalg.solve(H, b)
    f = lambda x: 0.5 * float(x @ H @ x) - float(b @ x)
    gr = lambda x: H @ x - b
    x0 = np.zeros(n)
    st = O.LBFGSState(x=x0, f=f(x0), g=gr(x0))
    for _ in range(300):
        O.lbfgs_step(st, f, gr, history=5)
    assert np.linalg.norm(st.x - xs) < 1e-7 * np.linalg.norm(xs)


def test_lbfgs_failed_search_keeps_x():
    """A function that never decreases enough: x is unchanged, history cleared, LS_FAIL."""
    x0 = np.ones(3)
    f = lambda x: 1.0 if np.array_equal(x, x0) else 2.0
    gr = lambda x: np.ones_like(x)
    st = O.LBFGSState(x=x0.copy(), f=f(x0), g=gr(x0), hist_s=[np.ones(3)], hist_y=[np.ones(3)])
    assert not O.lbfgs_step(st, f, gr, max_bt=6)
    assert np.array_equal(st.x, x0) and st.hist_s == [] and st.status & O.ST_LS_FAIL
    assert st.trials == 6


def test_lbfgs_block_on_the_loss_meets_armijo_every_step():
    """On the distillation loss itself (fixed V_c): every accepted step satisfies
    f(x + t d) <= f(x) + c1 t g.d with the g.d of a descent direction, so f never
    rises inside an L-BFGS block; checked against f and g recomputed from scratch."""
    Q, Kz, Vz, Kc, _ = tiny(n_q=40, z=20, k=5, d=8, seed=21)
    Y, lse = O.targets(Q, Kz, Vz)
    V, _ = O.ridge_fit(Q, Kc, Y, 1e-3)
    d = Q.shape[1]
    fl = lambda x: O.loss_only(Q, x.reshape(-1, d), V, Y, lse)
    fg = lambda x: O.loss_grad(Q, x.reshape(-1, d), V, Y, lse)[1].ravel()
    f0, g0, _ = O.loss_grad(Q, Kc, V, Y, lse)
    st = O.LBFGSState(x=Kc.ravel().copy(), f=f0, g=g0.ravel())
    for _ in range(8):
        x_old, f_old, g_old = st.x.copy(), st.f, st.g.copy()
        assert O.lbfgs_step(st, fl, fg)
        step = st.x - x_old
        assert float(g_old @ step) < 0.0                      # a descent step
        assert st.f <= f_old + 1e-4 * float(g_old @ step)     # Armijo with t d = step
        assert abs(st.f - fl(st.x)) <= 1e-12 * max(1.0, abs(st.f))
        np.testing.assert_allclose(st.g, fg(st.x), rtol=1e-10, atol=1e-14)


def test_ridge_fit_minimises_the_penalised_objective():
    """The fitted V_c is the minimiser of |A V - Y|^2 + lam |V|^2: random
    perturbations of either sign raise the objective by exactly |A E|^2 + lam |E|^2
    (a quadratic with zero gradient at the minimiser)."""
    Q, Kz, Vz, Kc, _ = tiny(n_q=30, z=12, k=5, d=6, seed=22)
    Y, lse = O.targets(Q, Kz, Vz)
    lam = 0.05
    V, _ = O.ridge_fit(Q, Kc, Y, lam)
    A, _ = O.attention(Q, Kc)
    obj = lambda W: float(np.sum((A @ W - Y) ** 2) + lam * np.sum(W ** 2))
    base = obj(V)
    r = np.random.default_rng(5)
    for _ in range(5):
        E = r.standard_normal(V.shape) * 1e-2
        for sgn in (1.0, -1.0):
            rise = obj(V + sgn * E) - base
            expect = float(np.sum((A @ E) ** 2) + lam * np.sum(E ** 2))
            assert abs(rise - expect) <= 1e-9 * max(1.0, base)


def test_compress_trace_and_select_fit():
    """Loss never rises across L-BFGS blocks followed by value re-fits in this
    small case, iteration 0 is Select+Fit, and the solve beats it."""
    Q, Kz, Vz, _, _ = tiny(n_q=48, z=24, d=8, seed=15)
    sched = O.Schedule(outer=6, steps=5)
    r = O.compress(Q, Kz, Vz, 6, sched)
    Y, lse = O.targets(Q, Kz, Vz)
    idx = O.topk_select(O.importance(Q, Kz, lse), 6)
    V0, _ = O.ridge_fit(Q, Kz[idx], Y, sched.lam)
    assert abs(r["trace"][0] - O.loss_only(Q, Kz[idx], V0, Y, lse)) < 1e-15
    assert np.all(np.diff(r["trace"]) <= 1e-15)
    assert r["loss"] < 0.5 * r["trace"][0]


# ------------------------------------------------------------- allocation

def test_allocation_golden(golden_dir):
    with open(os.path.join(golden_dir, "allocation_cases.json")) as fh:
        cases = json.load(fh)["cases"]
    for c in cases:
        got = O.pilot_allocate(c["mse"], c["total"], c["k_min"], c["k_max"], c["alpha"])
        assert got.tolist() == c["expect"], c["why"]


def _shares_by_bisection(w, lo, hi, total):
    a, b = 0.0, 1.0
    while np.minimum(hi, np.maximum(lo, b * w)).sum() < total:
        b *= 2
    for _ in range(200):
        c = 0.5 * (a + b)
        if np.minimum(hi, np.maximum(lo, c * w)).sum() < total:
            a = c
        else:
            b = c
    return np.minimum(hi, np.maximum(lo, b * w))


@pytest.mark.parametrize("seed", range(12))
def test_allocation_brute_force(seed):
    r = np.random.default_rng(100 + seed)
    B = int(r.integers(2, 5))
    k_min = int(r.integers(1, 4))
    k_max = r.integers(k_min + 1, 15, size=B)
    total = int(r.integers(B * k_min, int(k_max.sum()) + 1))
    mse = np.exp(r.uniform(-5, 5, size=B))
    got = O.pilot_allocate(mse, total, k_min, k_max, 0.5)
    ideal = _shares_by_bisection(np.sqrt(mse), np.full(B, float(k_min)), k_max.astype(float), total)
    best, best_cost = None, None
    for cand in itertools.product(*[range(k_min, int(k_max[b]) + 1) for b in range(B)]):
        if sum(cand) != total:
            continue
        cost = float(((np.array(cand) - ideal) ** 2).sum())
        if best_cost is None or cost < best_cost - 1e-12:
            best, best_cost = cand, cost
    assert tuple(got) == best
    assert got.sum() == total and np.all(got >= k_min) and np.all(got <= k_max)


@pytest.mark.parametrize("seed", range(25))
def test_allocation_spends_the_whole_budget(seed):
    """The budget is redistributed, not reduced: the real shares sum to the
    total, sit inside their bounds and are proportional to MSE^0.5 wherever
    unclamped (compared with a bisection on the proportionality constant)."""
    r = np.random.default_rng(900 + seed)
    B = int(r.integers(5, 120))
    k_min = int(r.integers(1, 20))
    k_max = r.integers(k_min, 2000, size=B)
    total = int(r.integers(B * k_min, int(k_max.sum()) + 1))
    mse = np.exp(r.uniform(-8, 4, size=B))
    from oracle.kvsculpt import _clamped_shares
    w = np.sqrt(mse)
    lo, hi = np.full(B, float(k_min)), k_max.astype(float)
    x = _clamped_shares(w, lo, hi, float(total))
    assert abs(x.sum() - total) < 1e-6 * total
    np.testing.assert_allclose(x, _shares_by_bisection(w, lo, hi, total), rtol=1e-9, atol=1e-9)
    k = O.pilot_allocate(mse, total, k_min, k_max, 0.5)
    assert k.sum() == total and np.all(np.abs(k - x) < 1.0)


def test_allocation_zero_signal_absorbs_leftover():
    """Zero-MSE problems weigh 0; when the others are all at k_max the rest of
    the budget is shared evenly among the zero-MSE problems (hand-derived)."""
    k = O.pilot_allocate([0.0, 4.0, 0.0], 50, 5, [30, 10, 30], 0.5)
    assert k.tolist() == [20, 10, 20]
    k = O.pilot_allocate([0.0, 4.0, 0.0], 20, 5, [30, 10, 30], 0.5)
    assert k.tolist() == [5, 10, 5]


def test_ridge_non_finite_inputs():
    """A NaN in Y leaves the Gram matrix finite and the solution NaN
    (ST_NONFINITE); a NaN in Q makes the Gram matrix non-finite, which has no
    Cholesky factor (ST_NOT_PD)."""
    Q, _, _, Kc, Vc = tiny(n_q=9, k=3, d=4, seed=4)
    Y = np.random.default_rng(5).standard_normal((9, 4))
    Y[2, 1] = np.nan
    V, st = O.ridge_fit(Q, Kc, Y, 1e-3)
    assert V is None and st == O.ST_NONFINITE
    Q2 = Q.copy()
    Q2[0, 0] = np.nan
    V, st = O.ridge_fit(Q2, Kc, np.nan_to_num(Y), 1e-3)
    assert V is None and st == O.ST_NOT_PD


def test_lbfgs_non_finite_trial_is_rejected_and_flagged():
    x0 = np.array([1.0, -2.0])
    st = O.LBFGSState(x=x0.copy(), f=2.5, g=x0.copy())
    ok = O.lbfgs_step(st, lambda x: float("nan"), lambda x: x, max_bt=4)
    assert not ok and st.trials == 4
    assert st.status & O.ST_NONFINITE and st.status & O.ST_LS_FAIL
    np.testing.assert_array_equal(st.x, x0)
