"""Random-restart search on the GPU against the oracle's restarts from the same
keys (summary §4 "Optimizer Efficacy"); every step runs through the C ABI."""
import numpy as np
import pytest
import torch

import oracle as O
import workload as W
from gpu_common import Case

pytestmark = pytest.mark.gpu


def test_restarts_match_oracle():
    from kv_cache_compression_kvsculpt_b200 import restarts as RS
    wl = W.WORKLOADS["single_d64"].with_(outer=3)
    c = Case(wl)
    R = 3
    inits = W.restart_inits(np.diff(c.bt.z_off), c.k, R, seed=2)
    K = c.K
    sched = K.Schedule(outer=wl.outer, steps=wl.steps)
    res = RS.compress_restarts(wl.d, c.q_off, c.bt.z_off, c.k, c.Q, c.Kz, c.Vz, inits, sched)
    torch.cuda.synchronize()
    assert not res["status"].any()
    assert res["trace"].shape == (wl.outer + 1, R, c.bt.B)
    osched = O.Schedule(outer=wl.outer, steps=wl.steps)
    co = c.batch.c_off_h
    for b in range(c.bt.B):
        runs, best = O.restart_search(c.Qs[b], c.Zk[b], c.Zv[b], int(c.k[b]), osched,
                                      [inits[r, co[b]:co[b + 1]] for r in range(R)])
        for r in range(R):
            o = runs[r]
            assert abs(res["trace"][0, r, b] - o["trace"][0]) <= 1e-3 * o["trace"][0] + 1e-7
            assert res["loss"][r, b] <= 1.05 * o["loss"] + 1e-7, (r, b)
            assert res["loss"][r, b] <= res["trace"][0, r, b]
            gi = res["idx"][(r * c.batch.sum_c + co[b]):(r * c.batch.sum_c + co[b + 1])]
            assert np.array_equal(gi.cpu().numpy(), inits[r, co[b]:co[b + 1]])
        assert res["best"][b] == int(np.argmin(res["loss"][:, b]))
