"""Host logic of the multi-GPU path on CPU: contiguous cost-balanced problem
blocks per rank, and the one collective of the adaptive budget (the all-gather
of pilot MSEs and zone sizes) run as two gloo ranks.  Every rank must reach
the allocation a single process computes over all problems ("KVSculpt: KV
Cache Compression as Distillation", section 2 "Adaptive Budget Allocation":
the budget is pooled over layers and heads)."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import kv_cache_compression_kvsculpt_b200 as K
from kv_cache_compression_kvsculpt_b200 import adaptive, shard


def test_partition_equal_costs_gives_equal_blocks():
    assert shard.partition(np.ones(56), 8) == [(7 * r, 7 * r + 7) for r in range(8)]
    assert shard.partition(np.ones(56), 1) == [(0, 56)]


def test_partition_covers_and_balances():
    r = np.random.default_rng(3)
    for world in (2, 3, 4, 8):
        costs = r.uniform(0.2, 5.0, 57)
        blocks = shard.partition(costs, world)
        assert blocks[0][0] == 0 and blocks[-1][1] == 57
        assert all(a[1] == b[0] for a, b in zip(blocks, blocks[1:]))
        assert all(e > s for s, e in blocks)
        sums = [costs[s:e].sum() for s, e in blocks]
        # no block exceeds its fair share by more than one problem's cost
        assert max(sums) <= costs.sum() / world + costs.max() + 1e-9


def test_partition_fewer_problems_than_ranks():
    blocks = shard.partition(np.ones(3), 4)
    assert blocks[0][0] == 0 and blocks[-1][1] == 3
    assert sum(e - s for s, e in blocks) == 3


def test_problem_cost_orders_by_work():
    c = shard.problem_cost([3840, 3840], [576, 1344], 128)
    assert c[1] > c[0]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, mse, z, counts, total, out):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        off = int(np.sum(counts[:rank]))
        sl = slice(off, off + counts[rank])
        k_loc, k_all, mse_all = adaptive.allocate_global(mse[sl], z[sl], total, 16, 0.5,
                                                         dist.group.WORLD)
        out[rank] = (k_loc.tolist(), k_all.tolist(), mse_all.tolist())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("counts", [(28, 28), (20, 36)])
def test_adaptive_allocation_over_two_gloo_ranks(counts):
    r = np.random.default_rng(sum(counts))
    B = sum(counts)
    mse = r.lognormal(-6, 1.0, B).astype(np.float32)
    z = np.full(B, 1920, np.int32)
    total = 960 * B
    want = K.kvs_pilot_allocate(mse, total, 16, z, 0.5)
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        ps = [ctx.Process(target=_rank_main, args=(rk, 2, port, mse, z, counts, total, out))
              for rk in range(2)]
        for p in ps:
            p.start()
        for p in ps:
            p.join(timeout=120)
        assert all(p.exitcode == 0 for p in ps)
        res = dict(out)
    assert sum(res[0][0]) + sum(res[1][0]) == total
    for rk in range(2):
        k_loc, k_all, mse_all = res[rk]
        np.testing.assert_array_equal(k_all, want)
        np.testing.assert_array_equal(mse_all, mse)
    np.testing.assert_array_equal(np.concatenate([res[0][0], res[1][0]]), want)
