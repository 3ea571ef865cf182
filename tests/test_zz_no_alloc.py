"""kvs_loss_grad_static: the loss/gradient call that allocates nothing.

Callers that cannot call cudaMalloc (a plug-in whose host application owns
all device memory, or a service whose device footprint is fixed at load time)
cannot hand kvs_loss_grad a workspace; kvs_loss_grad_static takes its scratch
from an array compiled into the library instead.  These tests call it through
the C ABI and compare it with kvs_loss_grad on the same inputs, twice in a row
with different keys (the shared array keeps the previous call's contents), at
the tolerance of the other loss/gradient tests.  The file is named to run
last, so a failure here cannot hide the result of any other test.
"""
import numpy as np
import pytest
import torch

import workload as W
from gpu_common import Case, cosine, dev, host

pytestmark = pytest.mark.gpu


def _point(c, seed):
    r = np.random.default_rng(seed)
    Kc = np.concatenate([c.Zk[b][:int(c.k[b])] for b in range(c.bt.B)]).astype(np.float64)
    Kc = (Kc + 0.2 * r.standard_normal(Kc.shape)).astype(np.float32)
    Vc = r.standard_normal(Kc.shape).astype(np.float32) * 0.1
    Y = r.standard_normal(c.Q.shape).astype(np.float32) * 0.05
    lse = (5.0 + r.standard_normal(c.Q.shape[0])).astype(np.float32)
    return dev(Kc), dev(Vc), dev(Y), dev(lse)


@pytest.mark.parametrize("name", ["single_d64", "ragged"])
def test_static_matches_workspace_call_twice(name):
    assert torch.cuda.is_available()
    if name == "single_d64":
        c = Case(W.WORKLOADS["single_d64"])
    else:
        wl = W.Workload("ragged_small", 1, 3, 2, d=128, N=300, m=44, g=2, n_syn=61, k=64,
                        layer_scale=True, outer=3, steps=4)
        c = Case(wl, k=[37, 100, 1, 256, 64, 129], n_q=[210, 173, 97, 210, 150, 201])
    K = c.K
    assert K.kvs_workspace_bytes(c.batch) <= 32 << 20
    B = c.bt.B
    for call in range(2):
        Kc, Vc, Y, lse = _point(c, seed=call)
        ref_loss = torch.empty(B, device="cuda")
        ref_parts = torch.empty((B, 2), device="cuda")
        ref_dK = torch.empty_like(Kc)
        K.kvs_loss_grad(c.batch, c.Q, Kc, Vc, Y, lse, 1.0, 1.0, ref_loss, ref_parts, ref_dK, c.ws)
        loss = torch.full((B,), float("nan"), device="cuda")
        parts = torch.full((B, 2), float("nan"), device="cuda")
        dK = torch.full_like(Kc, float("nan"))
        K.kvs_loss_grad_static(c.batch, c.Q, Kc, Vc, Y, lse, 1.0, 1.0, loss, parts, dK)
        torch.cuda.synchronize()
        if call == 1:
            # the call itself allocates no device memory: after a first call has
            # loaded the library's kernels, the free device memory does not move
            free0 = torch.cuda.mem_get_info()[0]
            K.kvs_loss_grad_static(c.batch, c.Q, Kc, Vc, Y, lse, 1.0, 1.0, loss, parts, dK)
            torch.cuda.synchronize()
            assert torch.cuda.mem_get_info()[0] == free0
        rl, l = host(ref_loss), host(loss)
        assert np.all(np.abs(l - rl) <= 1e-3 * np.abs(rl)), (call, l, rl)
        np.testing.assert_allclose(host(parts), host(ref_parts), rtol=1e-3, atol=1e-9)
        co = c.batch.c_off_h
        gd, rd = host(dK), host(ref_dK)
        for b in range(B):
            assert cosine(gd[co[b]:co[b + 1]], rd[co[b]:co[b + 1]]) >= 0.999, (call, b)


def test_static_rejects_batches_beyond_its_array():
    assert torch.cuda.is_available()
    c = Case(W.WORKLOADS["qwen_layer"])  # both KV heads of one layer
    K = c.K
    assert K.kvs_workspace_bytes(c.batch) > 32 << 20
    Kc = torch.zeros((c.batch.sum_c, c.wl.d), device="cuda")
    loss = torch.empty(c.bt.B, device="cuda")
    with pytest.raises(K.KvsError) as e:
        K.kvs_loss_grad_static(c.batch, c.Q, Kc, Kc, c.Q, c.Q[:, 0].contiguous(), 1.0, 1.0,
                               loss, None, None)
    assert e.value.rc == -4
