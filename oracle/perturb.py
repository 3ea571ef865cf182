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

__all__ = ["noisy_evaluations", "GPU_LEVELS"]

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
