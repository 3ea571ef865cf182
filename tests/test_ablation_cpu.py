"""Adam ablation (CPU): pins of the oracle's Adam step against closed-form facts,
the Adam schedule's consistency with the solve, and the C ABI's argument checks
for kvs_adam_step (summary §4 "Optimizer Efficacy")."""
import ctypes

import numpy as np
import pytest

import oracle as O


def test_adam_first_step_moves_by_lr_times_sign():
    # with zero moments the bias-corrected first step is g / |g| per coordinate
    g = np.array([3.0, -2e-3, 0.5, -7.0])
    x = np.zeros(4)
    x1, m, v = O.adam_step(x, g, np.zeros(4), np.zeros(4), 1, lr=0.01, eps=1e-12)
    np.testing.assert_allclose(x1, -0.01 * np.sign(g), rtol=1e-9)
    np.testing.assert_allclose(m, 0.1 * g)
    np.testing.assert_allclose(v, 0.001 * g * g)


def test_adam_is_invariant_to_gradient_scale():
    r = np.random.default_rng(8)
    x = r.standard_normal(6)
    m = v = np.zeros(6)
    xs, ms, vs = x.copy(), m.copy(), v.copy()
    for t in range(1, 6):
        g = r.standard_normal(6)
        x, m, v = O.adam_step(x, g, m, v, t, 0.05, eps=1e-14)
        xs, ms, vs = O.adam_step(xs, 1000.0 * g, ms, vs, t, 0.05, eps=1e-14)
    np.testing.assert_allclose(xs, x, rtol=1e-10, atol=1e-12)


def test_adam_constant_gradient_takes_lr_steps():
    # a constant gradient keeps m_hat = g and v_hat = g^2 at every t
    x = np.array([1.0, -1.0])
    m = v = np.zeros(2)
    g = np.array([0.3, -4.0])
    for t in range(1, 8):
        x, m, v = O.adam_step(x, g, m, v, t, 0.1, eps=0.0)
    np.testing.assert_allclose(x, np.array([1.0, -1.0]) - 7 * 0.1 * np.sign(g), rtol=1e-12)


def test_adam_compress_shares_the_select_fit_point_and_descends():
    r = np.random.default_rng(41)
    Q = r.standard_normal((30, 4))
    Kz = r.standard_normal((12, 4))
    Vz = r.standard_normal((12, 4))
    sched = O.Schedule(outer=3, steps=5)
    lb = O.compress(Q, Kz, Vz, 4, sched)
    ad = O.adam_compress(Q, Kz, Vz, 4, sched, lr=1e-2)
    assert ad["trace"][0] == lb["trace"][0]          # the same Select+Fit start
    assert np.array_equal(ad["idx"], lb["idx"])
    assert ad["loss"] < ad["trace"][0]
    tiny = O.adam_compress(Q, Kz, Vz, 4, sched, lr=1e-12)
    assert abs(tiny["loss"] - tiny["trace"][0]) < 1e-9 * tiny["trace"][0]


def test_adam_step_argument_errors(K=None):
    import kv_cache_compression_kvsculpt_b200 as K
    b = K.KvsBatch.uniform(2, 128, 40, 30, 7, device="cpu")
    fake = ctypes.c_void_p(1 << 20)   # aligned, never dereferenced on error paths
    lib = K.lib
    ok = (b.ref, fake, fake, fake, fake)
    assert lib.kvs_adam_step(*ok, 0, 1e-2, 0.9, 0.999, 1e-8, None) != 0      # t < 1
    assert lib.kvs_adam_step(*ok, 1, 0.0, 0.9, 0.999, 1e-8, None) != 0       # lr <= 0
    assert lib.kvs_adam_step(*ok, 1, 1e-2, 1.0, 0.999, 1e-8, None) != 0      # beta1 = 1
    assert lib.kvs_adam_step(*ok, 1, 1e-2, 0.9, -0.1, 1e-8, None) != 0       # beta2 < 0
    assert lib.kvs_adam_step(*ok, 1, 1e-2, 0.9, 0.999, 0.0, None) != 0       # eps <= 0
    assert lib.kvs_adam_step(b.ref, None, fake, fake, fake, 1, 1e-2, 0.9, 0.999, 1e-8, None) != 0
    unaligned = ctypes.c_void_p((1 << 20) + 4)
    assert lib.kvs_adam_step(b.ref, fake, unaligned, fake, fake, 1, 1e-2, 0.9, 0.999, 1e-8,
                             None) != 0


def test_adam_moments_persist_across_refits():
    """One Adam step per outer iteration: the first step moves every key
    coordinate by exactly lr (zero moments, bias correction), while the second,
    taken after the value re-fit with the moments carried over, does not."""
    r = np.random.default_rng(43)
    Q = r.standard_normal((20, 4))
    Kz = r.standard_normal((9, 4))
    Vz = r.standard_normal((9, 4))
    one = O.adam_compress(Q, Kz, Vz, 3, O.Schedule(outer=1, steps=1), lr=1e-2, eps=1e-14)
    two = O.adam_compress(Q, Kz, Vz, 3, O.Schedule(outer=2, steps=1), lr=1e-2, eps=1e-14)
    K0 = Kz[one["idx"]]
    np.testing.assert_allclose(np.abs(one["Kc"] - K0), 1e-2, rtol=1e-9)
    step2 = np.abs(two["Kc"] - one["Kc"])
    assert np.abs(step2 - 1e-2).max() > 1e-4
