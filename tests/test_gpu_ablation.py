"""Adam ablation on the GPU against the oracle (summary §4 "Optimizer Efficacy"):
the kvs_adam_step kernel on given moments and gradient, and the whole Adam
schedule through the C ABI."""
import numpy as np
import pytest
import torch

import oracle as O
import workload as W
from gpu_common import Case, dev, host

pytestmark = pytest.mark.gpu


def test_adam_step_kernel_matches_oracle():
    import kv_cache_compression_kvsculpt_b200 as K
    b = K.KvsBatch(128, [0, 40, 80], [0, 30, 60], [0, 7, 20])
    r = np.random.default_rng(17)
    n = (b.sum_c, 128)
    x = r.standard_normal(n).astype(np.float32)
    g = r.standard_normal(n).astype(np.float32)
    m = (0.1 * r.standard_normal(n)).astype(np.float32)
    v = (0.01 + 0.1 * r.random(n)).astype(np.float32)
    X, G, M, V = dev(x), dev(g), dev(m), dev(v)
    # the parameters as the kernel sees them (float32)
    lr, b1, b2, eps = (float(np.float32(p)) for p in (1e-2, 0.9, 0.999, 1e-8))
    K.kvs_adam_step(b, X, G, M, V, 3, lr, b1, b2, eps)
    torch.cuda.synchronize()
    xo, mo, vo = O.adam_step(x.astype(np.float64), g.astype(np.float64), m.astype(np.float64),
                             v.astype(np.float64), 3, lr, b1, b2, eps)
    np.testing.assert_allclose(host(M), mo, rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(host(V), vo, rtol=1e-6, atol=1e-9)
    step_gpu = host(X).astype(np.float64) - x
    np.testing.assert_allclose(step_gpu, xo - x, rtol=2e-4, atol=2e-7)


def test_adam_schedule_matches_oracle():
    from kv_cache_compression_kvsculpt_b200 import ablation as AB
    wl = W.WORKLOADS["single_d64"].with_(outer=2)
    c = Case(wl)
    K = c.K
    sched = K.Schedule(outer=wl.outer, steps=wl.steps)
    r = AB.compress_adam(c.batch, c.Q, c.Kz, c.Vz, sched, lr=1e-2)
    assert not r["status"].any()
    osched = O.Schedule(outer=wl.outer, steps=wl.steps)
    for b in range(c.bt.B):
        o = O.adam_compress(c.Qs[b], c.Zk[b], c.Zv[b], int(c.k[b]), osched, lr=1e-2)
        assert abs(r["trace"][0, b] - o["trace"][0]) <= 1e-3 * o["trace"][0] + 1e-7
        assert abs(r["trace"][-1, b] - o["loss"]) <= 0.05 * o["loss"] + 1e-7, (r["trace"][:, b],
                                                                                o["trace"])
