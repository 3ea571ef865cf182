"""Shared helpers of the GPU tests: seeded problems as oracle (float64 numpy)
and device (float32 torch) tensors of the same values."""
import numpy as np
import torch

import oracle as O
import workload as W


def dev(x, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(x)).to(device="cuda", dtype=dtype)


def host(t):
    return t.detach().cpu().numpy()


def rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def cosine(a, b):
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b)))


def oracle_queries(wl, bt):
    """Training queries of every problem by the oracle (float64 list)."""
    out = []
    for b in range(bt.B):
        p = bt.problem(b)
        out.append(O.build_queries(p["q_retain"], p["q_ctx"], p["pos"], wl.g, wl.m_q, wl.n_syn,
                                   wl.N, wl.rope_base))
    return out


class Case:
    """A batch of problems with fp32 inputs shared by both sides.

    Q is the oracle's training-query set rounded to float32, so per-step
    parity tests compare the two sides on identical inputs.
    """

    def __init__(self, wl, ids=None, seed=0, k=None, n_q=None):
        import kv_cache_compression_kvsculpt_b200 as K
        self.K = K
        self.wl = wl
        self.bt = W.make_batch(wl, seed, ids)
        B = self.bt.B
        self.Qs = [q.astype(np.float32) for q in oracle_queries(wl, self.bt)]
        if n_q is not None:  # ragged query counts: keep the first n_q[b] rows
            self.Qs = [q[:int(n)] for q, n in zip(self.Qs, n_q)]
        q_off = np.concatenate([[0], np.cumsum([len(q) for q in self.Qs])]).astype(np.int64)
        self.Zk = [self.bt.problem(b)["Kz"] for b in range(B)]
        self.Zv = [self.bt.problem(b)["Vz"] for b in range(B)]
        kk = np.broadcast_to(np.asarray(wl.k if k is None else k), (B,)).astype(np.int64)
        self.k = kk
        self.q_off = q_off
        self.batch = K.KvsBatch(wl.d, q_off, self.bt.z_off,
                                np.concatenate([[0], np.cumsum(kk)]))
        self.Q = dev(np.concatenate(self.Qs))
        self.Kz = dev(self.bt.Kz)
        self.Vz = dev(self.bt.Vz)
        self.ws = K.alloc_workspace(self.batch)

    def rows(self, t, off, b):
        return t[off[b]:off[b + 1]]

    def targets_oracle(self, b):
        return O.targets(self.Qs[b], self.Zk[b], self.Zv[b])


# Final-loss parity of the whole (non-convex, fixed-length) schedule.  The
# oracle's run is repeated with its loss and gradient evaluations perturbed at
# the relative precision of the library's arithmetic (oracle.perturb); the
# final losses of those runs and of the exact run span a band that arithmetic
# of that precision can legitimately reach.  The GPU's final loss must lie
# within 5 % of that band.  A trajectory whose band spans more than a factor
# 1.25 is ill-conditioned (a tiny change of the arithmetic sends it elsewhere):
# there the result is only required to improve on Select+Fit.
ILL_CONDITIONED = 0.25


def final_loss_bar(f_or, band, bar=0.05):
    """(low, high, spread) of the accepted final losses."""
    vals = [float(f_or)] + [float(v) for v in band]
    lo, hi = min(vals), max(vals)
    return lo * (1 - bar), hi * (1 + bar), hi / lo - 1.0


def oracle_band(Q, Kz, Vz, k, sched, seeds=3):
    """Final losses of the oracle's schedule with perturbed evaluations."""
    from oracle.perturb import GPU_LEVELS, noisy_evaluations
    return [float(O.compress(Q, Kz, Vz, k, sched, evaluate=noisy_evaluations(*GPU_LEVELS, s))
                  ["loss"]) for s in range(seeds)]


def check_final_loss(f_gpu, f_sf, f_or, band, what="", emulated=None):
    """Assert the parity bar above; returns 'ok', 'ok (emulated)' or 'ill-conditioned'.
    `emulated`: the final loss of the oracle's run with the library's own rounding
    emulated (oracle.perturb.emulated_evaluations), a member of the band when
    given; 'ok (emulated)' says the result needed it."""
    lo, hi, spread = final_loss_bar(f_or, band)
    if emulated is not None and not (lo - 1e-7 <= f_gpu <= hi + 1e-7):
        lo2, hi2, spread2 = final_loss_bar(f_or, list(band) + [emulated])
        if spread2 <= ILL_CONDITIONED:
            assert lo2 - 1e-7 <= f_gpu <= hi2 + 1e-7, (what, f_gpu, f_or, band, emulated,
                                                       f_gpu / f_or)
            return "ok (emulated)"
    if spread > ILL_CONDITIONED:
        assert f_gpu < f_sf, (what, f_gpu, f_sf)
        return "ill-conditioned"
    assert lo - 1e-7 <= f_gpu <= hi + 1e-7, (what, f_gpu, f_or, band, f_gpu / f_or)
    return "ok"
