"""L-BFGS with a populated history: the CUDA path against the oracle's two-loop
recursion and line search from the same stored pairs.

"KVSculpt: KV Cache Compression as Distillation", summary section 2 "Key
Optimization": the keys are optimised by L-BFGS.  The library evaluates the
two-loop recursion in inner-product form over a ring of (s, y) pairs kept on
the device; a slip in the ring's slot arithmetic or in the stored inner
products would only slow convergence, so the whole-schedule tests could miss
it.  Here, after a few steps through the C ABI, the state buffer is read back
(kvs_lbfgs_state_layout) and

* every stored pair is checked against the keys and gradients read after each
  step (s = x_new - x_old, y = g_new - g_old, bit for bit: both sides form the
  same float32 differences), newest pair in slot head - 1;
* the direction of the next step equals the oracle's two-loop recursion on the
  same g and pairs (float64), and the step taken equals the oracle's
  lbfgs_step started from the same x, f, g and pairs.
With history 3 the ring wraps around, so pairs are overwritten and the stored
inner products are reused across ring rotations.
"""
import numpy as np
import pytest
import torch

import oracle as O
import workload as W
from gpu_common import Case, host, rel
from test_gpu_parity import RAGGED, RAGGED_K, RAGGED_NQ, select_fit_point

pytestmark = pytest.mark.gpu

CASES = {
    "single_d64": lambda: Case(W.WORKLOADS["single_d64"]),
    "ragged": lambda: Case(RAGGED, k=RAGGED_K, n_q=RAGGED_NQ),
    "qwen_layer": lambda: Case(W.WORKLOADS["qwen_layer"]),
}


def read_state(K, c, state, history):
    """Per problem: x, g, f, dir and the stored pairs (oldest first) from the buffer."""
    L = K.kvs_lbfgs_state_layout(c.batch, history)
    raw = host(state).view(np.uint8)
    n = c.batch.sum_c * c.wl.d
    vec = lambda off: raw[off:off + 4 * n].view(np.float32)
    x, g, dr = vec(L["x"]), vec(L["g"]), vec(L["dir"])
    out = []
    co = c.batch.c_off_h
    for b in range(c.bt.B):
        rec = raw[L["scalars"] + b * L["scalar_bytes"]:][:L["scalar_bytes"]]
        f = float(rec[L["off_f"]:L["off_f"] + 4].view(np.float32)[0])
        count = int(rec[L["off_count"]:L["off_count"] + 4].view(np.int32)[0])
        head = int(rec[L["off_head"]:L["off_head"] + 4].view(np.int32)[0])
        s0, s1 = co[b] * c.wl.d, co[b + 1] * c.wl.d
        hs, hy = [], []
        for p in range(count - 1, -1, -1):  # oldest first
            slot = (head - 1 - p) % L["slots"]
            o_s = L["ring_s"] + slot * L["ring_stride"]
            o_y = L["ring_y"] + slot * L["ring_stride"]
            hs.append(raw[o_s:o_s + 4 * n].view(np.float32)[s0:s1].copy())
            hy.append(raw[o_y:o_y + 4 * n].view(np.float32)[s0:s1].copy())
        out.append(dict(x=x[s0:s1].copy(), g=g[s0:s1].copy(), dir=dr[s0:s1].copy(), f=f,
                        count=count, hist_s=hs, hist_y=hy))
    return out


@pytest.mark.parametrize("history", [10, 3])
@pytest.mark.parametrize("name", ["single_d64", "ragged", "qwen_layer"])
def test_step_from_a_populated_history(name, history):
    c = CASES[name]()
    K = c.K
    d = c.wl.d
    Kcs, Vcs, tgt = select_fit_point(c, perturb=0.3, seed=1)
    sched = K.Schedule(outer=1, steps=1, history=history)
    Y = torch.from_numpy(np.concatenate([t[0] for t in tgt])).cuda()
    lse = torch.from_numpy(np.concatenate([t[1] for t in tgt])).cuda()
    Vc = torch.from_numpy(np.concatenate(Vcs)).cuda()
    Kc = torch.from_numpy(np.concatenate(Kcs)).cuda()
    state = K.alloc_state(c.batch, history)
    status = torch.zeros(c.bt.B, dtype=torch.int32, device="cuda")
    K.kvs_lbfgs_reset(c.batch, sched, c.Q, Y, lse, Vc, Kc, state, 1, c.ws)
    snaps = [read_state(K, c, state, history)]
    n_before = 4
    for _ in range(n_before):
        K.kvs_lbfgs_step(c.batch, sched, c.Q, Y, lse, Vc, Kc, state, status, None, c.ws)
        snaps.append(read_state(K, c, state, history))
    assert not host(status).any()
    before = snaps[-1]
    # the 5th step
    fout = torch.empty(c.bt.B, device="cuda")
    K.kvs_lbfgs_step(c.batch, sched, c.Q, Y, lse, Vc, Kc, state, status, fout, c.ws)
    after = read_state(K, c, state, history)
    torch.cuda.synchronize()
    assert not host(status).any()
    gk, gf = host(Kc), host(fout)
    co = c.batch.c_off_h
    checked_pairs = 0
    for b in range(c.bt.B):
        st = before[b]
        # every step here was accepted (clean status); the pair of step j joins
        # iterates j and j+1 and is stored when it passes the curvature test
        cand = [(snaps[j + 1][b]["x"] - snaps[j][b]["x"], snaps[j + 1][b]["g"] - snaps[j][b]["g"])
                for j in range(n_before)]
        kept = [(s_, y_) for s_, y_ in cand
                if float(s_.astype(np.float64) @ y_) > 1e-10 * float(y_.astype(np.float64) @ y_)]
        kept = kept[-history:]
        assert st["count"] == len(kept), (b, st["count"], len(kept))
        for p, (s_want, y_want) in enumerate(kept):
            np.testing.assert_array_equal(st["hist_s"][p], s_want)
            np.testing.assert_array_equal(st["hist_y"][p], y_want)
            checked_pairs += 1
        # the direction: the oracle's two-loop recursion on the same g and pairs
        hs = [h.astype(np.float64) for h in st["hist_s"]]
        hy = [h.astype(np.float64) for h in st["hist_y"]]
        g64 = st["g"].astype(np.float64)
        d_or = O.two_loop_direction(g64, hs, hy)
        if not float(g64 @ d_or) < 0.0:
            d_or = -g64
        assert rel(after[b]["dir"], d_or) < 1e-4, (b, rel(after[b]["dir"], d_or))
        # the step: the oracle's lbfgs_step from the same x, f, g and pairs
        Q, Yo, lo, V = c.Qs[b], tgt[b][0], tgt[b][1], Vcs[b]
        ost = O.LBFGSState(x=st["x"].astype(np.float64), f=st["f"], g=g64,
                           hist_s=list(hs), hist_y=list(hy))
        ok = O.lbfgs_step(ost, lambda x: O.loss_only(Q, x.reshape(-1, d), V, Yo, lo),
                          lambda x: O.loss_grad(Q, x.reshape(-1, d), V, Yo, lo)[1].ravel(),
                          history=history)
        assert ok, b
        step_gpu = gk[co[b]:co[b + 1]].ravel().astype(np.float64) - st["x"]
        step_or = ost.x - st["x"]
        tol = 2e-2 * np.linalg.norm(step_or) + 2.0 ** -22 * np.linalg.norm(st["x"])
        assert np.linalg.norm(step_gpu - step_or) <= tol, (b, np.linalg.norm(step_gpu - step_or),
                                                           np.linalg.norm(step_or))
        assert abs(gf[b] - ost.f) <= 1e-3 * ost.f + 1e-7, (b, gf[b], ost.f)
    assert checked_pairs >= c.bt.B
