"""Property-based pins of the float64 oracle (hypothesis, CPU): the identities of
the pinned example tests, over random small shapes and seeds."""
import numpy as np
from hypothesis import given, settings, strategies as st

import oracle as O

SETTINGS = settings(max_examples=25, deadline=None, derandomize=True)
shapes = st.tuples(st.integers(1, 6), st.integers(1, 5), st.sampled_from([2, 4, 6]),
                   st.integers(0, 2 ** 31 - 1))


def _rand(n_q, k, d, seed, scale=1.0):
    r = np.random.default_rng(seed)
    return (r.standard_normal((n_q, d)) * scale, r.standard_normal((k, d)) * scale,
            r.standard_normal((k, d)), r)


@SETTINGS
@given(shapes, st.integers(1, 5))
def test_lse_merge_over_any_split(shape, k2):
    """Attention over [K1; K2] equals the LSE-weighted merge of the two chunks."""
    n_q, k1, d, seed = shape
    Q, K1, V1, r = _rand(n_q, k1, d, seed)
    K2 = r.standard_normal((k2, d))
    V2 = r.standard_normal((k2, d))
    Y, l = O.targets(Q, np.vstack([K1, K2]), np.vstack([V1, V2]))
    Y1, l1 = O.targets(Q, K1, V1)
    Y2, l2 = O.targets(Q, K2, V2)
    m = np.maximum(l1, l2)
    lm = m + np.log(np.exp(l1 - m) + np.exp(l2 - m))
    np.testing.assert_allclose(l, lm, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(Y, np.exp(l1 - lm)[:, None] * Y1 + np.exp(l2 - lm)[:, None] * Y2,
                               rtol=1e-10, atol=1e-12)


@SETTINGS
@given(shapes)
def test_gradient_matches_central_differences(shape):
    n_q, k, d, seed = shape
    Q, Kc, Vc, r = _rand(n_q, k, d, seed)
    Y = r.standard_normal((n_q, d))
    lse = r.standard_normal(n_q)
    f, g, _ = O.loss_grad(Q, Kc, Vc, Y, lse)
    assert abs(f - O.loss_only(Q, Kc, Vc, Y, lse)) <= 1e-12 * max(1.0, f)
    h = 1e-6
    num = np.zeros_like(Kc)
    for i in range(k):
        for j in range(d):
            E = np.zeros_like(Kc)
            E[i, j] = h
            num[i, j] = (O.loss_only(Q, Kc + E, Vc, Y, lse) - O.loss_only(Q, Kc - E, Vc, Y, lse)) / (2 * h)
    np.testing.assert_allclose(g, num, rtol=1e-5, atol=1e-8)


@SETTINGS
@given(st.lists(st.integers(0, 3), min_size=1, max_size=9), st.integers(1, 9))
def test_topk_equals_sorting_rule(vals, k):
    """Top-k of small integer scores (many ties): the k best by (-score, index), ascending."""
    k = min(k, len(vals))
    imp = np.array(vals, np.float64)
    ranked = sorted(range(len(vals)), key=lambda j: (-vals[j], j))
    got = O.topk_select(imp, k)
    assert list(got) == sorted(ranked[:k])
    # every chosen score is >= every unchosen one
    rest = [j for j in range(len(vals)) if j not in set(got)]
    assert all(imp[c] >= imp[u] for c in got for u in rest)


@SETTINGS
@given(shapes, st.sampled_from([1e-3, 1e-1, 1.0]))
def test_ridge_solves_its_normal_equations(shape, lam):
    n_q, k, d, seed = shape
    Q, Kc, _, r = _rand(n_q, k, d, seed)
    Y = r.standard_normal((n_q, d))
    V, st_ = O.ridge_fit(Q, Kc, Y, lam)
    assert st_ == O.ST_OK
    A, _ = O.attention(Q, Kc)
    res = (A.T @ A + lam * np.eye(k)) @ V - A.T @ Y
    assert np.linalg.norm(res) <= 1e-10 * max(1.0, np.linalg.norm(A.T @ Y))
