"""Adaptive budget: a pilot solve at uniform k, the allocation by pilot MSE,
then the full solve at the allocated sizes.

"KVSculpt: KV Cache Compression as Distillation", section 2 "Adaptive Budget
Allocation": a short pilot run measures how hard each head-problem is to
compress and the pooled budget follows its output MSE.  Every step runs in
the library: the pilot and the full solve are kvs_compress_batch calls and
the allocation is kvs_pilot_allocate (host C).  This module only sequences
the calls and sizes the buffers.  With a process group, each rank holds its
own problems; the ranks exchange pilot MSEs and zone sizes with one
all-gather and all compute the same allocation.
"""
from __future__ import annotations

import numpy as np
import torch

from . import _lib as L
from . import shard


def allocate_global(mse_loc, z_loc, total: int, k_min: int = 16, alpha: float = 0.5, group=None):
    """The pooled allocation from this rank's pilot MSEs and zone sizes: one
    all-gather of both, kvs_pilot_allocate over every problem (the same result
    on every rank), then this rank's slice.  Returns (k_local, k_all, mse_all)."""
    counts = shard.allgather_host(np.array([len(mse_loc)], np.int64), group)
    mse_all = shard.allgather_host(np.asarray(mse_loc, np.float32), group)
    z_all = shard.allgather_host(np.asarray(z_loc, np.int32), group)
    k_all = L.kvs_pilot_allocate(mse_all, int(total), int(k_min), z_all, float(alpha))
    rank = 0 if group is None else torch.distributed.get_rank(group)
    return shard.local_slice(k_all, counts, rank).astype(np.int64), np.asarray(k_all), mse_all


def compress_adaptive(d, q_off, z_off, Q, Kz, Vz, total: int, sched: L.Schedule,
                      pilot: L.Schedule, k_min: int = 16, alpha: float = 0.5, group=None,
                      stream=None):
    """Q [sum_q, d], Kz / Vz [sum_z, d] (CUDA, fp32) for this rank's problems
    with host offsets q_off, z_off.  `total` is the budget summed over the
    problems of every rank.  Returns a dict with the local Kc, Vc, c_off, k,
    loss trace, parts, status, and the global pilot MSE and allocation."""
    q_off = np.asarray(q_off, np.int64)
    z_off = np.asarray(z_off, np.int64)
    B = len(q_off) - 1
    dev = Q.device
    counts = shard.allgather_host(np.array([B], np.int64), group)
    z_loc = np.diff(z_off)
    k_uni = int(total) // int(counts.sum())
    if k_uni < 1 or np.any(k_uni > z_loc):
        raise ValueError("uniform pilot size must lie in [1, z_b] for every problem")

    def solve(k_loc, sc):
        batch = L.KvsBatch(d, q_off, z_off, np.concatenate([[0], np.cumsum(k_loc)]), device=dev)
        Kc = torch.empty((batch.sum_c, d), device=dev)
        Vc = torch.empty_like(Kc)
        trace = torch.empty((B, sc.outer + 1), device=dev)
        parts = torch.empty((B, 2), device=dev)
        status = torch.empty(B, dtype=torch.int32, device=dev)
        ws = L.alloc_workspace(batch, sc, device=dev)
        state = L.alloc_state(batch, sc.history, device=dev)
        L.kvs_compress_batch(batch, sc, Q, Kz, Vz, Kc, Vc, None, trace, parts, status, state, ws,
                             stream)
        return dict(batch=batch, Kc=Kc, Vc=Vc, trace=trace, parts=parts, status=status)

    pil = solve(np.full(B, k_uni, np.int64), pilot)
    mse_loc = pil["parts"][:, 0].float().cpu().numpy()  # output-MSE term after the pilot
    k_loc, k_all, mse_all = allocate_global(mse_loc, z_loc, total, k_min, alpha, group)
    full = solve(k_loc, sched)
    return dict(Kc=full["Kc"], Vc=full["Vc"], c_off=full["batch"].c_off_h, k=k_loc,
                trace=full["trace"], parts=full["parts"], status=full["status"],
                pilot_mse=mse_all, k_all=k_all, pilot_status=pil["status"])
