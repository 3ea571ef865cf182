"""Problem sharding over ranks (one process per GPU).

Head-problems are independent ("KVSculpt: KV Cache Compression as
Distillation", section 2: every layer and KV head is distilled on its own), so
a batch is cut into contiguous blocks, one per rank, with no exchange during
the solve.  The only collective is the all-gather of per-problem scalars that
the adaptive budget needs (section 2 "Adaptive Budget Allocation": the budget
is pooled over all layers and heads).  Host logic only; the collectives run on
whatever backend the process group has (NCCL on GPUs, gloo in CPU tests).
"""
from __future__ import annotations

import numpy as np


def problem_cost(n_q, k, d):
    """Relative cost of one head-problem: the loss/gradient contractions
    (n_q k d) plus the Gram matrix (n_q k^2)."""
    n_q = np.asarray(n_q, np.float64)
    k = np.asarray(k, np.float64)
    return n_q * k * d + n_q * k * k


def partition(costs, world: int):
    """Contiguous blocks [start_r, end_r) of problems, one per rank, that
    balance the summed cost: block r ends at the first problem whose prefix
    sum reaches (r + 1) / world of the total.  Every rank gets at least one
    problem when there are at least `world` problems."""
    c = np.asarray(costs, np.float64)
    B = len(c)
    if world < 1:
        raise ValueError("world must be >= 1")
    pre = np.concatenate([[0.0], np.cumsum(c)])
    tot = pre[-1]
    bounds = [0]
    for r in range(1, world):
        if tot > 0:
            e = int(np.searchsorted(pre, tot * r / world, side="left"))
        else:
            e = (B * r) // world
        lo = bounds[-1] + (1 if B - bounds[-1] > world - r else 0)
        hi = B - (world - r)  # leave one problem per later rank when possible
        e = min(max(e, lo), max(hi, lo))
        bounds.append(min(e, B))
    bounds.append(B)
    return [(bounds[r], bounds[r + 1]) for r in range(world)]


def allgather_host(values, group=None):
    """Concatenate every rank's 1-D host array in rank order (all ranks get
    the same result).  Without a process group the input comes back."""
    a = np.ascontiguousarray(np.asarray(values))
    if group is None:
        return a
    import torch.distributed as dist
    world = dist.get_world_size(group)
    parts = [None] * world
    dist.all_gather_object(parts, a, group=group)
    return np.concatenate(parts)


def local_slice(global_values, counts, rank: int):
    """This rank's part of an array gathered by allgather_host, given every
    rank's problem count in rank order."""
    off = int(np.sum(counts[:rank]))
    return np.asarray(global_values)[off:off + int(counts[rank])]
