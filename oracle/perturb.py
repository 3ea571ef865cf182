"""Perturbed loss and gradient evaluations for the oracle's schedule (test
infrastructure only: used to measure how sensitive a trajectory is, never by the
library).

The alternating schedule is a fixed-length run of a non-convex optimiser
("KVSculpt: KV Cache Compression as Distillation", summary section 2
"Optimization Strategy"), so where it ends can depend on rounding: a line
search that accepts or halves on a loss difference below the arithmetic's
precision, or a curvature pair built from a slightly different gradient, sends
the rest of the run elsewhere.  `noisy_evaluations(level_f, level_g, seed)`
returns replacements for oracle.loss_only / oracle.loss_grad whose results are
multiplied by (1 + level * noise), the noise drawn from a generator seeded by
a hash of the evaluation point and `seed` (so a run is reproducible), uniform
in [-1, 1] for the loss and standard normal per gradient element.  Running
oracle.compress with them at the levels of the GPU arithmetic (about 16
significant bits in every product) shows the spread of final losses that
arithmetic of that precision can reach.
"""
from __future__ import annotations

import hashlib

import numpy as np

from .kvsculpt import loss_grad, loss_only

__all__ = ["noisy_evaluations", "GPU_LEVELS", "emulated_evaluations"]

# relative levels of the library's arithmetic: the loss carries about 2^-16 of
# its largest terms (measured near 1e-6 relative), the gradient about 5e-4 in
# norm at an optimised point (cosine 1 - 1.2e-7 in the precision study)
GPU_LEVELS = (2e-6, 5e-4)


def _rng(x, seed):
    h = hashlib.blake2b(np.ascontiguousarray(x, np.float64).tobytes() + seed.to_bytes(4, "little"),
                        digest_size=8).digest()
    return np.random.default_rng(int.from_bytes(h, "little"))


def noisy_evaluations(level_f: float, level_g: float, seed: int):
    def f_only(Q, Kc, Vc, Y, lse, w_out=1.0, w_lse=1.0):
        f = loss_only(Q, Kc, Vc, Y, lse, w_out, w_lse)
        return f * (1.0 + level_f * (_rng(Kc, seed).random() * 2.0 - 1.0))

    def f_grad(Q, Kc, Vc, Y, lse, w_out=1.0, w_lse=1.0):
        f, g, info = loss_grad(Q, Kc, Vc, Y, lse, w_out, w_lse)
        r = _rng(Kc, seed)
        f = f * (1.0 + level_f * (r.random() * 2.0 - 1.0))
        return f, g * (1.0 + level_g * r.standard_normal(g.shape)), info

    return f_only, f_grad


# ---------------------------------------------------------------------------
# The library's own rounding, emulated in float64.  Every product of the loss
# and gradient takes its operands as bf16 pairs x = hi + lo and forms
# hi.hi + hi.lo + lo.hi (about 16 significant bits); dL/dY_hat enters the
# value product of the gradient as fp16 scaled by a power of two into fp16's
# normal range, and delta is formed from the same rounded values.  A run with
# these evaluations shows where a fixed-length solve with that arithmetic ends
# on a given trajectory.
# ---------------------------------------------------------------------------

def _bf16(x):
    x = np.ascontiguousarray(np.asarray(x, np.float32))
    v = x.view(np.uint32).copy()
    v = v + np.uint32(0x7FFF) + ((v >> np.uint32(16)) & np.uint32(1))
    v &= np.uint32(0xFFFF0000)
    return v.view(np.float32).astype(np.float64)


def _split(x):
    x32 = np.asarray(x, np.float32).astype(np.float64)
    hi = _bf16(x32)
    return hi, _bf16(x32 - hi)


def _mm3(a, b):
    ah, al = _split(a)
    bh, bl = _split(b)
    return ah @ bh + ah @ bl + al @ bh


def _emulated_loss_grad(Q, Kc, Vc, Y, lse, w_out=1.0, w_lse=1.0, need_grad=True):
    Q = np.asarray(Q, np.float64)
    Kc = np.asarray(Kc, np.float64)
    Vc = np.asarray(Vc, np.float64)
    Y = np.asarray(Y, np.float64)
    lse = np.asarray(lse, np.float64)
    n_q, d = Q.shape
    s = 1.0 / np.sqrt(d)
    S = _mm3(Q, Kc.T) * s
    mx = S.max(axis=1, keepdims=True)
    l_h = mx[:, 0] + np.log(np.exp(S - mx).sum(axis=1))
    A = np.exp(S - l_h[:, None])
    Yh = _mm3(A, Vc)
    out = float(((Yh - Y) ** 2).sum()) / (n_q * d)
    ls = float(((l_h - lse) ** 2).sum()) / n_q
    f = w_out * out + w_lse * ls
    if not need_grad:
        return f, None, dict(out=out, lse=ls)
    c = 2.0 * w_out / (n_q * d)
    sig = 2.0 ** -np.rint(np.log2(c)) if c > 0 else 1.0
    G = np.asarray(c * sig * (Yh - Y), np.float32).astype(np.float16).astype(np.float64) / sig
    delta = (G * Yh).sum(axis=1) - (2.0 * w_lse / n_q) * (l_h - lse)
    dS = A * (G @ Vc.T - delta[:, None])
    return f, _mm3(dS.T, Q) * s, dict(out=out, lse=ls)


def emulated_evaluations():
    """Replacements for loss_only / loss_grad with the library's rounding (above)."""
    def f_only(Q, Kc, Vc, Y, lse, w_out=1.0, w_lse=1.0):
        return _emulated_loss_grad(Q, Kc, Vc, Y, lse, w_out, w_lse, need_grad=False)[0]

    def f_grad(Q, Kc, Vc, Y, lse, w_out=1.0, w_lse=1.0):
        return _emulated_loss_grad(Q, Kc, Vc, Y, lse, w_out, w_lse)

    return f_only, f_grad
