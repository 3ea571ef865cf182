"""Batched random-restart search over the initial keys.

"KVSculpt: KV Cache Compression as Distillation", summary §4 "Optimizer
Efficacy": a single L-BFGS run from the top-k keys is compared with the best of
100 random restarts.  Here R restarts of B head-problems run as one batch of
R * B problems on the library's kernels (problem order: restart-major).
Restart r of problem b starts from k_b zone keys the caller chooses (the
search's random subsets, e.g. ``workload.restart_inits``), takes their ridge
values and runs the alternating schedule: `steps` L-BFGS steps on K_c, a ridge
re-fit of V_c, `outer` times.  Every step runs in the library through its C
ABI; this module only lays out the replicated batch and picks, per problem,
the restart with the lowest final loss.

The chosen subsets enter through ``kvs_init_topk``: an importance vector that
is 1 at the chosen zone positions and 0 elsewhere makes the top-k selection
return exactly those keys (ascending), gathered on the device.

Run as ``python -m kv_cache_compression_kvsculpt_b200.restarts`` to compare the
single top-k run with the best of R restarts on a synthetic workload and to
time the search (one JSON line).
"""
from __future__ import annotations

import numpy as np
import torch

from . import _lib as K


def replicate_offsets(off, restarts: int) -> np.ndarray:
    """Row offsets of `restarts` back-to-back copies of a batch with offsets `off`."""
    counts = np.diff(np.asarray(off, np.int64))
    return np.concatenate([[0], np.cumsum(np.tile(counts, restarts))]).astype(np.int64)


def init_mask(z_off, c_off, inits) -> np.ndarray:
    """Importance [R * sum z] that is 1 at the zone positions inits[r] chooses for
    every problem and 0 elsewhere (inits: int [R, sum k], problem b's entries at
    c_off[b] .., each a set of k_b distinct positions in [0, z_b))."""
    z_off = np.asarray(z_off, np.int64)
    c_off = np.asarray(c_off, np.int64)
    inits = np.asarray(inits)
    R, B = inits.shape[0], len(z_off) - 1
    sz = int(z_off[-1])
    imp = np.zeros(R * sz, np.float32)
    for r in range(R):
        for b in range(B):
            z = int(z_off[b + 1] - z_off[b])
            pos = inits[r, c_off[b]:c_off[b + 1]].astype(np.int64)
            if len(np.unique(pos)) != len(pos) or pos.min() < 0 or pos.max() >= z:
                raise ValueError(f"restart {r}, problem {b}: positions must be distinct, in [0, {z})")
            imp[r * sz + z_off[b] + pos] = 1.0
    return imp


def compress_restarts(d: int, q_off, z_off, k, Q, Kz, Vz, inits, sched: K.Schedule,
                      stream=None):
    """Run the schedule from each restart's keys for every problem of the batch.

    Q [sum q, d], Kz / Vz [sum z, d]: device float32 tensors of the B problems;
    k: int or per-problem list; inits: int [R, sum k] zone positions.  Returns a
    dict with `trace` [outer + 1, R, B] (loss after every fit), `loss` [R, B],
    `best` [B] (restart of the lowest final loss, the first on ties), `status`
    [R, B], and the device tensors `Kc`, `Vc` [R * sum k, d] and `idx` [R * sum k].
    """
    dev = Q.device
    B = len(q_off) - 1
    kk = np.broadcast_to(np.asarray(k, np.int64), (B,))
    c_off = np.concatenate([[0], np.cumsum(kk)]).astype(np.int64)
    inits = np.asarray(inits)
    R = inits.shape[0]
    if inits.ndim != 2 or inits.shape[1] != c_off[-1]:
        raise ValueError("inits must be [restarts, sum k]")
    base = K.KvsBatch(d, q_off, z_off, c_off, device=dev)
    Y = torch.empty_like(Q)
    lse = torch.empty(base.sum_q, device=dev)
    K.kvs_targets(base, Q, Kz, Vz, Y, lse, None, K.alloc_workspace(base, device=dev), stream)

    rep = K.KvsBatch(d, replicate_offsets(q_off, R), replicate_offsets(z_off, R),
                     replicate_offsets(c_off, R), device=dev)
    Qr, Yr, lr = Q.repeat(R, 1), Y.repeat(R, 1), lse.repeat(R)
    Kzr = Kz.repeat(R, 1)
    imp = torch.from_numpy(init_mask(z_off, c_off, inits)).to(dev)
    idx = torch.empty(rep.sum_c, dtype=torch.int32, device=dev)
    Kc = torch.empty((rep.sum_c, d), device=dev)
    Vc = torch.empty_like(Kc)
    status = torch.zeros(R * B, dtype=torch.int32, device=dev)
    loss = torch.empty(R * B, device=dev)
    ws = K.alloc_workspace(rep, sched, device=dev)
    state = K.alloc_state(rep, sched.history, device=dev)
    trace = []

    def fit_and_restart(clear):
        K.kvs_fit_values(rep, Qr, Kc, Yr, sched.lam, Vc, status, ws, stream)
        K.kvs_lbfgs_reset(rep, sched, Qr, Yr, lr, Vc, Kc, state, clear, ws, stream)
        K.kvs_loss_grad(rep, Qr, Kc, Vc, Yr, lr, sched.w_out, sched.w_lse, loss, None, None, ws,
                        stream)
        trace.append(loss.clone())

    K.kvs_init_topk(rep, imp, Kzr, idx, Kc, stream)
    fit_and_restart(1)
    for _ in range(sched.outer):
        for _ in range(sched.steps):
            K.kvs_lbfgs_step(rep, sched, Qr, Yr, lr, Vc, Kc, state, status, None, ws, stream)
        fit_and_restart(0 if sched.persist_history else 1)
    tr = torch.stack(trace).cpu().numpy().reshape(len(trace), R, B)
    final = tr[-1]
    return {"trace": tr, "loss": final, "best": np.argmin(final, axis=0),
            "status": status.cpu().numpy().reshape(R, B), "Kc": Kc, "Vc": Vc, "idx": idx}


def _main():
    import argparse
    import json
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import workload as W

    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--workload", default="qwen_layer", choices=sorted(W.WORKLOADS))
    ap.add_argument("--problems", type=int, default=None, help="first n problems of the workload")
    ap.add_argument("--restarts", type=int, default=8)
    ap.add_argument("--seed", type=int, default=0)
    args = ap.parse_args()
    wl = W.WORKLOADS[args.workload]
    ids = wl.problem_ids()[:args.problems] if args.problems else None
    bt = W.make_batch(wl, args.seed, ids)
    dev = torch.device("cuda")
    t = lambda a, dt=torch.float32: torch.from_numpy(np.ascontiguousarray(a)).to(dev, dt)
    spec = K.QuerySpec(bt.B, wl.d, wl.g, wl.m_q, wl.n_syn, wl.N, wl.rope_base)
    Q = torch.empty((bt.B * wl.n_q, wl.d), device=dev)
    K.kvs_build_queries(spec, t(bt.q_retain), t(bt.q_ctx), t(bt.pos, torch.int32), Q)
    Kz, Vz = t(bt.Kz), t(bt.Vz)
    sched = K.Schedule(outer=wl.outer, steps=wl.steps, history=wl.history, lam=wl.lam,
                       w_out=wl.w_out, w_lse=wl.w_lse)
    # the single run from the top-k keys (the solve itself)
    batch = K.KvsBatch(wl.d, bt.q_off, bt.z_off, np.arange(bt.B + 1) * wl.k, device=dev)
    Kc1 = torch.empty((batch.sum_c, wl.d), device=dev)
    Vc1 = torch.empty_like(Kc1)
    tr1 = torch.empty((bt.B, wl.outer + 1), device=dev)
    st1 = torch.empty(bt.B, dtype=torch.int32, device=dev)
    K.kvs_compress_batch(batch, sched, Q, Kz, Vz, Kc1, Vc1, None, tr1, None, st1,
                         K.alloc_state(batch, sched.history, device=dev),
                         K.alloc_workspace(batch, device=dev))
    single = tr1[:, -1].cpu().numpy()
    inits = W.restart_inits(np.diff(bt.z_off), [wl.k] * bt.B, args.restarts, args.seed)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    res = compress_restarts(wl.d, bt.q_off, bt.z_off, wl.k, Q, Kz, Vz, inits, sched)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    best = res["loss"].min(axis=0)
    gap = single / best - 1.0
    print(json.dumps({
        "workload": args.workload, "problems": bt.B, "restarts": args.restarts,
        "schedule": f"{wl.outer}x{wl.steps}", "k": wl.k,
        "single_topk_loss": [float(x) for x in single],
        "best_of_restarts_loss": [float(x) for x in best],
        "single_over_best_minus_1": [round(float(x), 4) for x in gap],
        "restart_losses_median": [float(x) for x in np.median(res["loss"], axis=0)],
        "status_nonzero": int((res["status"] != 0).sum()),
        "search_ms": round(ms, 1),
        "restart_problems_per_s": round(args.restarts * bt.B / (ms * 1e-3), 2),
    }))


if __name__ == "__main__":
    _main()
