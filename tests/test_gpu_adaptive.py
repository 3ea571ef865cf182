"""Adaptive budget on the GPU ("KVSculpt: KV Cache Compression as
Distillation", section 2 "Adaptive Budget Allocation"): a pilot solve at
uniform k, the allocation by pilot output MSE, then the full solve at the
allocated sizes, through the library's calls.  Compared with the oracle on the
same float32 inputs: the allocation must be exactly the oracle's allocation of
the GPU's pilot MSEs (an integer result decided from the same floats), close
to the oracle's own allocation, and every full solve must reach the oracle's
loss at the same k within the usual 5 %."""
import numpy as np
import pytest

import oracle as O
import workload as W
from gpu_common import Case, host

pytestmark = pytest.mark.gpu

ADAPT = W.Workload("adaptive_small", 1, 3, 2, d=64, N=256, m=32, g=2, n_syn=48, k=64,
                   layer_scale=True, outer=4, steps=4, adaptive=True, pilot_outer=2,
                   pilot_steps=4)


def test_adaptive_small_matches_oracle():
    from kv_cache_compression_kvsculpt_b200 import adaptive
    c = Case(ADAPT)
    K, wl = c.K, c.wl
    B = c.bt.B
    total = wl.k * B
    z = np.diff(c.bt.z_off).astype(np.int64)
    sched = K.Schedule(outer=wl.outer, steps=wl.steps)
    pilot = K.Schedule(outer=wl.pilot_outer, steps=wl.pilot_steps)
    res = adaptive.compress_adaptive(wl.d, c.q_off, c.bt.z_off, c.Q, c.Kz, c.Vz, total, sched,
                                     pilot, k_min=16, alpha=0.5)
    assert not host(res["pilot_status"]).any() and not host(res["status"]).any()
    k = res["k"]
    assert k.sum() == total and np.all(k >= 16) and np.all(k <= z)
    want = O.pilot_allocate(res["pilot_mse"].astype(np.float64), total, 16, z, 0.5)
    np.testing.assert_array_equal(k, want)

    osched = O.Schedule(outer=wl.outer, steps=wl.steps)
    opilot = O.Schedule(outer=wl.pilot_outer, steps=wl.pilot_steps)
    probs = [dict(Q=c.Qs[b], Kz=c.Zk[b], Vz=c.Zv[b]) for b in range(B)]
    o = O.adaptive_compress(probs, total, osched, opilot, k_min=16, alpha=0.5)
    np.testing.assert_allclose(res["pilot_mse"], o["pilot_mse"], rtol=0.05)
    assert np.abs(k - o["k"]).sum() <= 0.05 * total

    trace = host(res["trace"])
    for b in range(B):
        r = O.compress(c.Qs[b], c.Zk[b], c.Zv[b], int(k[b]), osched)
        f_gpu = float(trace[b, -1])
        assert f_gpu <= 1.05 * r["loss"] + 1e-7, (b, f_gpu, r["loss"])
        assert f_gpu <= trace[b, 0]
