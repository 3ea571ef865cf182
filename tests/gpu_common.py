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
