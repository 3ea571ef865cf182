"""Optimiser ablation: Adam on the compressed keys in place of L-BFGS.

"KVSculpt: KV Cache Compression as Distillation", summary §4 "Optimizer
Efficacy": replacing L-BFGS by Adam leaves a much larger per-layer error.  This
module runs the same alternating schedule as the solve (top-k keys, ridge
values, then `outer` times { `steps` key updates; ridge re-fit }) with one Adam
step per loss/gradient evaluation; every step runs in the library through its
C ABI (kvs_loss_grad for the gradient, kvs_adam_step for the update).  The
moments and the step count persist across value re-fits.

Run as ``python -m kv_cache_compression_kvsculpt_b200.ablation`` to compare
the final losses of L-BFGS and Adam on a synthetic workload (one JSON line).
"""
from __future__ import annotations

import numpy as np
import torch

from . import _lib as K


def compress_adam(batch: K.KvsBatch, Q, Kz, Vz, sched: K.Schedule, lr: float, beta1=0.9,
                  beta2=0.999, eps=1e-8, stream=None):
    """Returns `trace` [outer + 1, B] (loss after every fit), `status` [B] and the
    device tensors `Kc`, `Vc`, `idx`."""
    dev = Q.device
    B, d = batch.B, batch.d
    ws = K.alloc_workspace(batch, sched, device=dev)
    Y = torch.empty_like(Q)
    lse = torch.empty(batch.sum_q, device=dev)
    imp = torch.empty(batch.sum_z, device=dev)
    K.kvs_targets(batch, Q, Kz, Vz, Y, lse, imp, ws, stream)
    idx = torch.empty(batch.sum_c, dtype=torch.int32, device=dev)
    Kc = torch.empty((batch.sum_c, d), device=dev)
    K.kvs_init_topk(batch, imp, Kz, idx, Kc, stream)
    Vc = torch.empty_like(Kc)
    status = torch.zeros(B, dtype=torch.int32, device=dev)
    loss = torch.empty(B, device=dev)
    dK = torch.empty_like(Kc)
    m = torch.zeros_like(Kc)
    v = torch.zeros_like(Kc)
    trace = []

    def fit():
        K.kvs_fit_values(batch, Q, Kc, Y, sched.lam, Vc, status, ws, stream)
        K.kvs_loss_grad(batch, Q, Kc, Vc, Y, lse, sched.w_out, sched.w_lse, loss, None, None, ws,
                        stream)
        trace.append(loss.clone())

    fit()
    t = 0
    for _ in range(sched.outer):
        for _ in range(sched.steps):
            t += 1
            K.kvs_loss_grad(batch, Q, Kc, Vc, Y, lse, sched.w_out, sched.w_lse, loss, None, dK,
                            ws, stream)
            K.kvs_adam_step(batch, Kc, dK, m, v, t, lr, beta1, beta2, eps, stream)
        fit()
    return {"trace": torch.stack(trace).cpu().numpy(), "status": status.cpu().numpy(),
            "Kc": Kc, "Vc": Vc, "idx": idx}


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
    ap.add_argument("--lr", type=float, nargs="+", default=[1e-3, 1e-2, 1e-1])
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
    batch = K.KvsBatch(wl.d, bt.q_off, bt.z_off, np.arange(bt.B + 1) * wl.k, device=dev)
    Kc1 = torch.empty((batch.sum_c, wl.d), device=dev)
    Vc1 = torch.empty_like(Kc1)
    tr1 = torch.empty((bt.B, wl.outer + 1), device=dev)
    st1 = torch.empty(bt.B, dtype=torch.int32, device=dev)
    K.kvs_compress_batch(batch, sched, Q, Kz, Vz, Kc1, Vc1, None, tr1, None, st1,
                         K.alloc_state(batch, sched.history, device=dev),
                         K.alloc_workspace(batch, device=dev))
    lbfgs = tr1.cpu().numpy()
    out = {"workload": args.workload, "problems": bt.B, "schedule": f"{wl.outer}x{wl.steps}",
           "k": wl.k, "select_fit_loss": [float(x) for x in lbfgs[:, 0]],
           "lbfgs_loss": [float(x) for x in lbfgs[:, -1]], "adam": []}
    for lr in args.lr:
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        r = compress_adam(batch, Q, Kz, Vz, sched, lr)
        e1.record()
        torch.cuda.synchronize()
        fin = r["trace"][-1]
        out["adam"].append({
            "lr": lr, "loss": [float(x) for x in fin],
            "adam_over_lbfgs": [round(float(a / b), 3) for a, b in zip(fin, lbfgs[:, -1])],
            "status_nonzero": int((r["status"] != 0).sum()),
            "ms": round(e0.elapsed_time(e1), 1)})
    print(json.dumps(out))


if __name__ == "__main__":
    _main()
