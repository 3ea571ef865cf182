"""Float64 restatement of each step of KVSculpt (test infrastructure only).

Citations name the page "KVSculpt: KV Cache Compression as Distillation" and
the section of it that defines the step ("Summary 2" is the structured
summary's section 2 "Methodology: KVSCULPT"; "Abstract" is the arXiv abstract).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import scipy.linalg

__all__ = [
    "ST_OK", "ST_NONFINITE", "ST_NOT_PD", "ST_LS_FAIL",
    "rope_inv_freq", "rope", "derope", "build_queries",
    "attention", "targets", "importance", "topk_select", "ridge_fit",
    "loss_grad", "loss_only", "two_loop_direction", "LBFGSState", "lbfgs_step",
    "Schedule", "compress", "restart_search", "adam_step", "adam_compress",
    "pilot_allocate", "adaptive_compress",
]

ST_OK = 0
ST_NONFINITE = 1
ST_NOT_PD = 2
ST_LS_FAIL = 4


# ---------------------------------------------------------------------------
# Rotary position embedding (Summary 1 "Problem Statement": pairs are compared
# after RoPE; Summary 2 "Training Query Construction": De-RoPE factorisation).
# Rotate-half pairing (i, i + d/2), theta_i = base^(-2 i / d).
# ---------------------------------------------------------------------------

def rope_inv_freq(d: int, base: float) -> np.ndarray:
    return base ** (-(np.arange(d // 2, dtype=np.float64) * 2.0) / d)


def _rotate(x: np.ndarray, positions: np.ndarray, base: float, sign: float) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[1]
    half = d // 2
    ang = np.asarray(positions, dtype=np.float64)[:, None] * rope_inv_freq(d, base)[None, :]
    c, s = np.cos(ang), sign * np.sin(ang)
    lo, hi = x[:, :half], x[:, half:]
    return np.concatenate([lo * c - hi * s, hi * c + lo * s], axis=1)


def rope(x, positions, base):
    """Rotate each row of x to its position."""
    return _rotate(x, positions, base, +1.0)


def derope(x, positions, base):
    """Inverse rotation: recovers the position-free content vector."""
    return _rotate(x, positions, base, -1.0)


def build_queries(q_retain, q_ctx, pos, g: int, m_q: int, n_syn: int, N: int, base: float):
    """Training query set of one KV-head problem (Summary 2 "Training Query Construction").

    1. Retain queries: the real queries of the retain zone, used as they are.
    2. Synthetic future queries: each sampled context query is de-RoPE'd at its
       own position (content extraction) and re-embedded at a future position;
       the j-th sampled query (ascending context position) of a query head goes
       to position N + j.
    Rows are ordered by query head, then retain rows, then synthetic rows.
    """
    q_retain = np.asarray(q_retain, np.float64).reshape(g, m_q, -1)
    q_ctx = np.asarray(q_ctx, np.float64).reshape(g, n_syn, -1)
    pos = np.asarray(pos).reshape(g, n_syn)
    fut = N + np.arange(n_syn)
    rows = []
    for h in range(g):
        content = derope(q_ctx[h], pos[h], base)
        rows.append(q_retain[h])
        rows.append(rope(content, fut, base))
    return np.concatenate(rows, axis=0)


# ---------------------------------------------------------------------------
# Attention over one chunk (Summary 2 "Problem Formulation" / "Loss Function").
# ---------------------------------------------------------------------------

def attention(Q, K):
    """Softmax weights A = exp(S - l) and row log-sum-exp l of S = Q K^T / sqrt(d)."""
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    S = (Q @ K.T) / math.sqrt(Q.shape[1])
    mx = S.max(axis=1, keepdims=True)
    lse = mx[:, 0] + np.log(np.exp(S - mx).sum(axis=1))
    A = np.exp(S - lse[:, None])
    return A, lse


def targets(Q, Kz, Vz):
    """Attention output Y and log-sum-exp l of the training queries over the compress zone."""
    A, lse = attention(Q, Kz)
    return A @ np.asarray(Vz, np.float64), lse


def importance(Q, Kz, lse):
    """Attention importance of each compress-zone position (Summary 2 "Initialization").

    imp_j = sum_i exp(S_ij - l_i): the attention probability the training queries
    put on key j, summed over all queries.
    """
    Q = np.asarray(Q, np.float64)
    S = (Q @ np.asarray(Kz, np.float64).T) / math.sqrt(Q.shape[1])
    return np.exp(S - np.asarray(lse, np.float64)[:, None]).sum(axis=0)


def topk_select(imp, k: int) -> np.ndarray:
    """Indices of the k most important positions, ties to the lower index, ascending."""
    imp = np.asarray(imp)
    order = sorted(range(len(imp)), key=lambda j: (-float(imp[j]), j))
    return np.array(sorted(order[:k]), dtype=np.int64)


def ridge_fit(Q, Kc, Y, lam: float):
    """Closed-form values (Summary 2 "Value Optimization"; Abstract).

    With the attention weights A induced by the current keys fixed,
    V_c = argmin ||A V - Y||_F^2 + lam ||V||_F^2 = (A^T A + lam I)^-1 A^T Y.
    Returns (V_c, status); a Gram matrix that is not positive definite gives
    ST_NOT_PD and V_c = None, and so does one with a non-finite entry (it has
    no Cholesky factor); a finite Gram matrix with a non-finite solution (e.g.
    a NaN in Y) gives ST_NONFINITE and V_c = None.
    """
    A, _ = attention(Q, Kc)
    G = A.T @ A + lam * np.eye(A.shape[1])
    R = A.T @ np.asarray(Y, np.float64)
    if not np.all(np.isfinite(G)):
        return None, ST_NOT_PD
    try:
        V = scipy.linalg.solve(G, R, assume_a="pos", check_finite=False)
    except np.linalg.LinAlgError:
        return None, ST_NOT_PD
    if not np.all(np.isfinite(V)):
        return None, ST_NONFINITE
    return V, ST_OK


def _loss_parts(Yh, Y, lse_h, lse):
    n_q, d = Y.shape
    out = float(((Yh - Y) ** 2).sum()) / (n_q * d)
    ls = float(((lse_h - lse) ** 2).sum()) / n_q
    return out, ls


def loss_only(Q, Kc, Vc, Y, lse, w_out=1.0, w_lse=1.0):
    """Distillation loss (Summary 2 "Loss Function"): output MSE + LSE MSE."""
    A, lse_h = attention(Q, Kc)
    Yh = A @ np.asarray(Vc, np.float64)
    out, ls = _loss_parts(Yh, np.asarray(Y, np.float64), lse_h, np.asarray(lse, np.float64))
    return w_out * out + w_lse * ls


def loss_grad(Q, Kc, Vc, Y, lse, w_out=1.0, w_lse=1.0):
    """Loss and its gradient with respect to the compressed keys.

    Y_hat = A V_c, l_hat = LSE(S), S = Q K_c^T / sqrt(d).
    dL/dY_hat = G = 2 w_out/(n_q d) (Y_hat - Y);  dL/dl_hat = gl = 2 w_lse/n_q (l_hat - l).
    Through the softmax: dL/dS_ij = A_ij (G_i . v_j - G_i . Y_hat_i + gl_i),
    and dL/dK_c = (dL/dS)^T Q / sqrt(d).
    Returns (f, grad, info) with info = dict(out=..., lse=...) unweighted terms.
    """
    Q = np.asarray(Q, np.float64)
    Y = np.asarray(Y, np.float64)
    Vc = np.asarray(Vc, np.float64)
    lse = np.asarray(lse, np.float64)
    n_q, d = Q.shape
    A, lse_h = attention(Q, Kc)
    Yh = A @ Vc
    out, ls = _loss_parts(Yh, Y, lse_h, lse)
    f = w_out * out + w_lse * ls
    G = (2.0 * w_out / (n_q * d)) * (Yh - Y)
    gl = (2.0 * w_lse / n_q) * (lse_h - lse)
    dP = G @ Vc.T
    delta = (G * Yh).sum(axis=1) - gl
    dS = A * (dP - delta[:, None])
    grad = (dS.T @ Q) / math.sqrt(d)
    return f, grad, dict(out=out, lse=ls)


# ---------------------------------------------------------------------------
# Key optimisation by L-BFGS (Summary 2 "Key Optimization"; Abstract).
# ---------------------------------------------------------------------------

def two_loop_direction(g, hist_s, hist_y):
    """Search direction -H g by the two-loop recursion (pairs oldest first).

    H0 = gamma I with gamma = s^T y / y^T y of the newest pair (1 without history).
    """
    q = np.array(g, dtype=np.float64, copy=True)
    n = len(hist_s)
    rho = [1.0 / float(hist_s[i] @ hist_y[i]) for i in range(n)]
    alpha = [0.0] * n
    for i in range(n - 1, -1, -1):
        alpha[i] = rho[i] * float(hist_s[i] @ q)
        q = q - alpha[i] * hist_y[i]
    gamma = 1.0
    if n:
        gamma = float(hist_s[-1] @ hist_y[-1]) / float(hist_y[-1] @ hist_y[-1])
    r = gamma * q
    for i in range(n):
        beta = rho[i] * float(hist_y[i] @ r)
        r = r + (alpha[i] - beta) * hist_s[i]
    return -r


@dataclass
class LBFGSState:
    x: np.ndarray                 # flattened keys
    f: float
    g: np.ndarray
    hist_s: list = field(default_factory=list)
    hist_y: list = field(default_factory=list)
    status: int = ST_OK
    trials: int = 0               # loss evaluations spent in line searches


def lbfgs_step(st: LBFGSState, fun_loss, fun_grad, history=10, c1=1e-4, backtrack=0.5,
               max_bt=20, curv_eps=1e-10):
    """One L-BFGS iteration with a deterministic backtracking Armijo line search.

    fun_loss(x) -> f;  fun_grad(x) -> g (both at the same fixed values V_c).
    Returns True when a step was accepted.
    """
    d = two_loop_direction(st.g, st.hist_s, st.hist_y)
    gtd = float(st.g @ d)
    if not gtd < 0.0:
        d = -st.g
        gtd = -float(st.g @ st.g)
    if st.hist_s:
        t = 1.0
    else:
        gn = float(np.sqrt(st.g @ st.g))
        t = min(1.0, 1.0 / gn) if gn > 0.0 else 1.0
    for _ in range(max_bt):
        xt = st.x + t * d
        ft = fun_loss(xt)
        st.trials += 1
        if not math.isfinite(ft):  # rejected below (a NaN comparison is false)
            st.status |= ST_NONFINITE
        if ft <= st.f + c1 * t * gtd:
            gt = fun_grad(xt)
            s = xt - st.x
            y = gt - st.g
            if float(s @ y) > curv_eps * float(y @ y):
                st.hist_s.append(s)
                st.hist_y.append(y)
                if len(st.hist_s) > history:
                    st.hist_s.pop(0)
                    st.hist_y.pop(0)
            st.x, st.f, st.g = xt, ft, gt
            return True
        t *= backtrack
    st.hist_s.clear()
    st.hist_y.clear()
    st.status |= ST_LS_FAIL
    return False


# ---------------------------------------------------------------------------
# The alternating schedule (Abstract: keys by L-BFGS, values in closed form,
# alternating every few steps; Summary 2 "Optimization Strategy").
# ---------------------------------------------------------------------------

@dataclass
class Schedule:
    outer: int = 40
    steps: int = 5
    history: int = 10
    lam: float = 1e-3
    w_out: float = 1.0
    w_lse: float = 1.0
    c1: float = 1e-4
    backtrack: float = 0.5
    max_bt: int = 20
    persist_history: bool = True


def compress(Q, Kz, Vz, k: int, sched: Schedule, idx: Optional[np.ndarray] = None,
             record: Optional[list] = None, evaluate=None):
    """Distil one compress zone (K_z, V_z) into k pairs for the training queries Q.

    targets -> importance -> top-k keys -> ridge values (Select+Fit state) ->
    [steps x L-BFGS on K_c, ridge re-fit of V_c] x outer.  Returns a dict with
    K_c, V_c, the loss trace after every fit (outer + 1 entries), the final
    loss terms, the top-k indices and the status bits.  When `record` is a
    list, a copy of (K_c, V_c, number of stored L-BFGS pairs) is appended to
    it after every fit (outer + 1 entries); nothing else changes.  `evaluate`
    (a pair of functions with the signatures of loss_only and loss_grad)
    replaces the loss and gradient evaluations that steer the schedule, e.g. by
    perturbed ones to measure how sensitive the trajectory is; the reported
    losses are still evaluated exactly.  Default: the plain ones.
    """
    ev_loss, ev_grad = evaluate if evaluate is not None else (loss_only, loss_grad)
    Q = np.asarray(Q, np.float64)
    d = Q.shape[1]
    Y, lse = targets(Q, Kz, Vz)
    if idx is None:
        idx = topk_select(importance(Q, Kz, lse), k)
    Kc = np.asarray(Kz, np.float64)[idx].copy()
    status = ST_OK
    Vc, st_fit = ridge_fit(Q, Kc, Y, sched.lam)
    status |= st_fit
    if Vc is None:
        Vc = np.zeros((len(idx), d))

    def fl(x):
        return ev_loss(Q, x.reshape(-1, d), Vc, Y, lse, sched.w_out, sched.w_lse)

    def fg(x):
        return ev_grad(Q, x.reshape(-1, d), Vc, Y, lse, sched.w_out, sched.w_lse)[1].ravel()

    f, g, _ = ev_grad(Q, Kc, Vc, Y, lse, sched.w_out, sched.w_lse)
    st = LBFGSState(x=Kc.ravel().copy(), f=f, g=g.ravel())
    trace = [loss_only(Q, Kc, Vc, Y, lse, sched.w_out, sched.w_lse) if evaluate else f]
    if record is not None:
        record.append((Kc.copy(), Vc.copy(), 0))
    for _o in range(sched.outer):
        for _t in range(sched.steps):
            lbfgs_step(st, fl, fg, sched.history, sched.c1, sched.backtrack, sched.max_bt)
        Kc = st.x.reshape(-1, d)
        V_new, st_fit = ridge_fit(Q, Kc, Y, sched.lam)
        status |= st_fit
        if V_new is not None:
            Vc = V_new
        if not sched.persist_history:
            st.hist_s.clear()
            st.hist_y.clear()
        f, g, _ = ev_grad(Q, Kc, Vc, Y, lse, sched.w_out, sched.w_lse)
        st.f, st.g = f, g.ravel()
        trace.append(loss_only(Q, Kc, Vc, Y, lse, sched.w_out, sched.w_lse) if evaluate else f)
        if record is not None:
            record.append((Kc.copy(), Vc.copy(), len(st.hist_s)))
    f, _, info = loss_grad(Q, Kc, Vc, Y, lse, sched.w_out, sched.w_lse)
    if not math.isfinite(f):
        status |= ST_NONFINITE
    return dict(Kc=Kc, Vc=Vc, trace=np.array(trace), loss=f, mse_out=info["out"],
                mse_lse=info["lse"], idx=np.asarray(idx), status=status | st.status,
                trials=st.trials, Y=Y, lse=lse)


# ---------------------------------------------------------------------------
# Adaptive budget allocation (Summary 2 "Adaptive Budget Allocation"; Abstract).
# ---------------------------------------------------------------------------


def restart_search(Q, Kz, Vz, k: int, sched: Schedule, inits):
    """Random-restart search over the initial keys ("KVSculpt: KV Cache Compression
    as Distillation", summary §4 "Optimizer Efficacy": a single L-BFGS run is
    compared with the best of 100 random restarts).  Each restart runs the whole
    schedule of `compress` from the zone keys inits[r] (k positions) instead of
    the top-k ones; returns the results and the index of the lowest final loss
    (the first one on ties)."""
    runs = [compress(Q, Kz, Vz, k, sched, idx=np.asarray(ix)) for ix in inits]
    losses = [r["loss"] for r in runs]
    return runs, int(np.argmin(losses))


def adam_step(x, g, m, v, t: int, lr: float, beta1=0.9, beta2=0.999, eps=1e-8):
    """One Adam step (Kingma & Ba, bias-corrected moments); returns (x, m, v)."""
    m = beta1 * m + (1.0 - beta1) * g
    v = beta2 * v + (1.0 - beta2) * g * g
    mh = m / (1.0 - beta1 ** t)
    vh = v / (1.0 - beta2 ** t)
    return x - lr * mh / (np.sqrt(vh) + eps), m, v


def adam_compress(Q, Kz, Vz, k: int, sched: Schedule, lr: float, beta1=0.9, beta2=0.999,
                  eps=1e-8, idx: Optional[np.ndarray] = None):
    """The schedule of `compress` with Adam on K_c in place of L-BFGS: the
    optimiser ablation of the page ("KVSculpt: KV Cache Compression as
    Distillation", summary §4 "Optimizer Efficacy").  `steps` Adam steps per
    outer iteration, one step per loss/gradient evaluation; the moments and the
    step count persist across value re-fits (one optimiser across outers)."""
    Q = np.asarray(Q, np.float64)
    d = Q.shape[1]
    Y, lse = targets(Q, Kz, Vz)
    if idx is None:
        idx = topk_select(importance(Q, Kz, lse), k)
    Kc = np.asarray(Kz, np.float64)[idx].copy()
    Vc, status = ridge_fit(Q, Kc, Y, sched.lam)
    if Vc is None:
        Vc = np.zeros((len(idx), d))
    trace = [loss_only(Q, Kc, Vc, Y, lse, sched.w_out, sched.w_lse)]
    m = np.zeros_like(Kc)
    v = np.zeros_like(Kc)
    t = 0
    for _o in range(sched.outer):
        for _s in range(sched.steps):
            t += 1
            _, g, _ = loss_grad(Q, Kc, Vc, Y, lse, sched.w_out, sched.w_lse)
            Kc, m, v = adam_step(Kc, g, m, v, t, lr, beta1, beta2, eps)
        V_new, st_fit = ridge_fit(Q, Kc, Y, sched.lam)
        status |= st_fit
        if V_new is not None:
            Vc = V_new
        trace.append(loss_only(Q, Kc, Vc, Y, lse, sched.w_out, sched.w_lse))
    return dict(Kc=Kc, Vc=Vc, trace=np.array(trace), loss=float(trace[-1]), idx=idx,
                status=status)

def _clamped_shares(w, lo, hi, total):
    """x_b = clip(c * w_b, lo_b, hi_b) with the scalar c >= 0 chosen so that sum x = total.

    sum_b x_b(c) is continuous, non-decreasing and linear between the
    breakpoints lo_b / w_b and hi_b / w_b, so c is found exactly on the
    segment that brackets the total.
    """
    def shares(c):
        return np.minimum(hi, np.maximum(lo, c * w))

    pos = w > 0
    cuts = np.unique(np.concatenate([lo[pos] / w[pos], hi[pos] / w[pos], [0.0]]))
    prev = 0.0
    for c in cuts:
        if shares(c).sum() >= total:
            break
        prev = c
    else:
        return shares(cuts[-1])
    base = shares(prev)
    mid = 0.5 * (prev + c)  # no breakpoint lies strictly inside (prev, c)
    free = pos & (mid * w > lo) & (mid * w < hi)
    slope = w[free].sum()
    if slope <= 0.0:
        return shares(c)
    cstar = prev + (total - base.sum()) / slope
    return shares(cstar)


def pilot_allocate(mse, total: int, k_min: int, k_max, alpha: float = 0.5) -> np.ndarray:
    """Redistribute a total budget of pairs in proportion to pilot MSE^alpha.

    The page gives the law (budget proportional to the square root of the pilot
    MSE, at layer and KV-head granularity); the bounds and the integer rounding
    are this restatement's reading: the real-valued shares are
    x_b = clip(c * MSE_b^alpha, k_min, k_max_b) with sum x_b = total (if the
    problems with a positive MSE cannot absorb the budget even at k_max, the
    zero-MSE problems share the remainder evenly), and the
    integers are floor(x_b) plus one unit for the largest fractional parts
    (ties to the lower problem index) until the total is met.
    """
    mse = np.asarray(mse, np.float64)
    B = len(mse)
    hi = np.broadcast_to(np.asarray(k_max, np.int64), (B,)).astype(np.float64)
    lo = np.full(B, float(k_min))
    if total < lo.sum() or total > hi.sum() or np.any(hi < lo):
        raise ValueError("budget outside [B*k_min, sum(k_max)]")
    w = np.where(np.isfinite(mse) & (mse > 0), mse, 0.0) ** alpha
    if w.sum() <= 0.0:
        w = np.ones(B)
    pos = w > 0
    if hi[pos].sum() + lo[~pos].sum() < total:
        # the problems with a positive signal cannot absorb the budget: they all get
        # k_max and the zero-signal problems share the rest evenly
        ideal = hi.copy()
        ideal[~pos] = _clamped_shares(np.ones(int((~pos).sum())), lo[~pos], hi[~pos],
                                      float(total - hi[pos].sum()))
    else:
        ideal = _clamped_shares(w, lo, hi, float(total))
    base = np.floor(ideal)
    frac = ideal - base
    k = base.astype(np.int64)
    left = int(total - k.sum())
    order = sorted(range(B), key=lambda b: (-frac[b], b))
    for b in order[:left]:
        k[b] += 1
    return k


def adaptive_compress(problems, total: int, sched: Schedule, pilot: Schedule, k_min=16,
                      alpha=0.5):
    """Pilot run at uniform k, allocation by pilot MSE, then the full solves.

    problems: list of dicts with Q, Kz, Vz.  The pilot signal is the output-MSE
    term after the pilot's last value fit.
    """
    B = len(problems)
    k_uni = total // B
    mse = []
    for p in problems:
        r = compress(p["Q"], p["Kz"], p["Vz"], k_uni, pilot)
        mse.append(r["mse_out"])
    kb = pilot_allocate(mse, total, k_min, [len(p["Kz"]) for p in problems], alpha)
    res = [compress(p["Q"], p["Kz"], p["Vz"], int(kb[b]), sched) for b, p in enumerate(problems)]
    return dict(pilot_mse=np.array(mse), k=kb, results=res)
