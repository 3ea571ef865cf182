"""The precision design, checked on the CPU (no GPU involved).

Every contraction of the CUDA path takes its operands as bf16 pairs x = hi + lo
and forms hi.hi + hi.lo + lo.hi with fp32 accumulation (about 16 significant
bits); the ridge system is factored in fp32.  This test emulates that
arithmetic in numpy (bf16 rounding to nearest even, products accumulated in
float64, which is closer to exact than the hardware's fp32 and so isolates the
operand rounding) on a Qwen-shaped problem at an optimised point, and checks it
against the float64 oracle with the parity bars of the GPU tests: loss within
rel 1e-3, gradient cosine >= 0.999, V_c within rel 1e-3.  Single-pass bf16
operands miss those bars at the same point, which is why the split is there.
"""
import numpy as np
import pytest
import scipy.linalg as sl

import oracle as O
import workload as W


def bf16(x):
    """Round float32 values to bf16 (nearest, ties to even); returned as float64."""
    x = np.ascontiguousarray(np.asarray(x, np.float32))
    v = x.view(np.uint32).copy()
    v = v + np.uint32(0x7FFF) + ((v >> np.uint32(16)) & np.uint32(1))
    v &= np.uint32(0xFFFF0000)
    return v.view(np.float32).astype(np.float64)


def split(x):
    x32 = np.asarray(x, np.float32).astype(np.float64)
    hi = bf16(x32)
    return hi, bf16(x32 - hi)


def mm_single(a, b):
    return bf16(a) @ bf16(b)


def mm_split(a, b):
    ah, al = split(a)
    bh, bl = split(b)
    return ah @ bh + ah @ bl + al @ bh


@pytest.fixture(scope="module")
def point():
    """One Qwen-shaped head subsampled to 640 queries and 480 zone keys, k = 160,
    solved for 4 x 5 steps by the oracle (an optimised point, where the loss is
    small and its gradient a small sum of large terms)."""
    wl = W.WORKLOADS["qwen_layer"]
    bt = W.make_batch(wl, 0, ids=[(0, 0, 0)])
    p = bt.problem(0)
    Q = O.build_queries(p["q_retain"], p["q_ctx"], p["pos"], wl.g, wl.m_q, wl.n_syn, wl.N,
                        wl.rope_base)
    Q = Q[::6].astype(np.float32).astype(np.float64)
    Kz = p["Kz"][::4].astype(np.float64)
    Vz = p["Vz"][::4].astype(np.float64)
    r = O.compress(Q, Kz, Vz, 160, O.Schedule(outer=4, steps=5))
    Y, lse = O.targets(Q, Kz, Vz)
    return Q, r["Kc"], r["Vc"], Y, lse


def loss_grad_emulated(mm, Q, Kc, Vc, Y, lse):
    s = 1.0 / np.sqrt(Q.shape[1])
    S = mm(Q, Kc.T) * s
    mx = S.max(1, keepdims=True)
    l = mx[:, 0] + np.log(np.exp(S - mx).sum(1))
    A = np.exp(S - l[:, None])
    Yh = mm(A, Vc)
    n_q, d = Q.shape
    f = ((Yh - Y) ** 2).sum() / (n_q * d) + ((l - lse) ** 2).sum() / n_q
    G = 2.0 / (n_q * d) * (Yh - Y)
    delta = (G * Yh).sum(1) - 2.0 / n_q * (l - lse)
    dS = A * (mm(G, Vc.T) - delta[:, None])
    return f, mm(dS.T, Q) * s


def fit_emulated(mm, Q, Kc, Y, lam=1e-3):
    s = 1.0 / np.sqrt(Q.shape[1])
    S = (mm(Q, Kc.T) * s).astype(np.float32).astype(np.float64)
    mx = S.max(1, keepdims=True)
    l = mx[:, 0] + np.log(np.exp(S - mx).sum(1))
    A = np.exp(S - l[:, None]).astype(np.float32).astype(np.float64)
    k = Kc.shape[0]
    G = mm(A.T, A).astype(np.float32) + np.float32(lam) * np.eye(k, dtype=np.float32)
    R = mm(A.T, Y).astype(np.float32)
    L = np.linalg.cholesky(G).astype(np.float32)  # fp32 factor and solves
    return sl.solve_triangular(L.T, sl.solve_triangular(L, R, lower=True), lower=False)


def _cos(a, b):
    return float((a * b).sum() / (np.linalg.norm(a) * np.linalg.norm(b)))


def test_split_operands_meet_the_loss_and_gradient_bars(point):
    Q, Kc, Vc, Y, lse = point
    f0, g0, _ = O.loss_grad(Q, Kc, Vc, Y, lse)
    f, g = loss_grad_emulated(mm_split, Q, Kc, Vc, Y, lse)
    assert abs(f - f0) <= 1e-5 * f0           # bar 1e-3
    assert _cos(g, g0) >= 0.99999             # bar 0.999
    f1, g1 = loss_grad_emulated(mm_single, Q, Kc, Vc, Y, lse)
    assert abs(f1 - f0) > 1e-3 * f0 or _cos(g1, g0) < 0.999   # one pass of bf16 does not


def test_split_gram_and_fp32_cholesky_meet_the_value_bar(point):
    Q, Kc, _, Y, _ = point
    Vo, _ = O.ridge_fit(Q, Kc, Y, 1e-3)
    rel = lambda V: float(np.linalg.norm(V - Vo) / np.linalg.norm(Vo))
    assert rel(fit_emulated(mm_split, Q, Kc, Y)) <= 1e-4   # bar 1e-3
    assert rel(fit_emulated(mm_single, Q, Kc, Y)) > 1e-3


def tf32(x, nearest=True):
    """float32 values kept to tf32's 10 mantissa bits: rounded to nearest (ties to
    even), or truncated, which is what the tensor cores do with the low bits of
    an fp32 operand they are handed as tf32."""
    x = np.ascontiguousarray(np.asarray(x, np.float32))
    v = x.view(np.uint32).copy()
    if nearest:
        v = v + np.uint32(0xFFF) + ((v >> np.uint32(13)) & np.uint32(1))
    v &= np.uint32(0xFFFFE000)
    return v.view(np.float32).astype(np.float64)


def test_single_pass_tf32_leaves_no_margin(point):
    """tf32 operands (the other input type the tensor cores take at fp32
    accumulation) in one pass: rounded to nearest they land just inside the
    gradient and value bars at the optimised point, with no margin for a full
    solve's steps to stay near the float64 trajectory; as the hardware truncates
    raw fp32 operands they miss the gradient bar."""
    Q, Kc, Vc, Y, lse = point
    f0, g0, _ = O.loss_grad(Q, Kc, Vc, Y, lse)
    Vo, _ = O.ridge_fit(Q, Kc, Y, 1e-3)
    rel = lambda V: float(np.linalg.norm(V - Vo) / np.linalg.norm(Vo))
    mm_rn = lambda a, b: tf32(a) @ tf32(b)
    mm_tr = lambda a, b: tf32(a, False) @ tf32(b, False)
    f, g = loss_grad_emulated(mm_rn, Q, Kc, Vc, Y, lse)
    assert abs(f - f0) <= 1e-3 * f0 and 0.999 <= _cos(g, g0) < 0.9995
    assert 5e-4 < rel(fit_emulated(mm_rn, Q, Kc, Y)) <= 1e-3
    _, g1 = loss_grad_emulated(mm_tr, Q, Kc, Vc, Y, lse)
    assert _cos(g1, g0) < 0.999


def f16(x):
    return np.asarray(x, np.float32).astype(np.float16).astype(np.float64)


def grad_with_go(Q, Kc, Vc, Y, lse, rnd):
    """Exact gradient except that dL/dY_hat is rounded by rnd before both the
    value product and delta (as in the key-gradient kernel)."""
    n_q, d = Q.shape
    A, l = O.attention(Q, Kc)
    Yh = A @ Vc
    G = rnd(2.0 / (n_q * d) * (Yh - Y))
    delta = (G * Yh).sum(1) - 2.0 / n_q * (l - lse)
    return ((A * (G @ Vc.T - delta[:, None])).T @ Q) / np.sqrt(d)


def test_go_in_scaled_fp16_beats_bf16(point):
    """Go = dL/dY_hat is the one operand that enters its product without a lo
    part.  In bf16 (8-bit mantissa) its rounding moves the gradient near an
    optimum by a few 1e-4, enough to steer some full-length solves several
    percent away from the float64 one; fp16 (11 bits) after scaling by a power
    of two into fp16's normal range moves it about eight times less, at the
    same MMA cost."""
    Q, Kc, Vc, Y, lse = point
    n_q, d = Q.shape
    _, g0, _ = O.loss_grad(Q, Kc, Vc, Y, lse)
    sig = 2.0 ** -np.rint(np.log2(2.0 / (n_q * d)))
    err = lambda g: float(np.linalg.norm(g - g0) / np.linalg.norm(g0))
    e_bf = err(grad_with_go(Q, Kc, Vc, Y, lse, bf16))
    e_f16 = err(grad_with_go(Q, Kc, Vc, Y, lse, lambda G: f16(G * sig) / sig))
    assert e_f16 <= e_bf / 4, (e_f16, e_bf)
    assert e_f16 < 1e-4


def test_emulated_evaluations_model_the_library_rounding(point):
    """oracle.perturb.emulated_evaluations (used to bound the final-loss parity
    bar) rounds like the library: close to the exact loss and gradient at the
    16-bit level, and not identical to them."""
    from oracle.perturb import emulated_evaluations
    Q, Kc, Vc, Y, lse = point
    f0, g0, _ = O.loss_grad(Q, Kc, Vc, Y, lse)
    fo, fg = emulated_evaluations()
    f1, g1, _ = fg(Q, Kc, Vc, Y, lse)
    assert abs(f1 - f0) <= 1e-5 * f0 and f1 != f0
    assert _cos(g1, g0) >= 0.99999 and not np.array_equal(g1, g0)
    assert fo(Q, Kc, Vc, Y, lse) == f1
