"""C-ABI checks that need no GPU: the library loads, exports every entry point
the header declares, sizes workspaces, rejects bad arguments before any
launch, and its host-only budget allocation matches the oracle exactly."""
import ctypes
import json
import os
import re

import numpy as np
import pytest

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvsculpt.h")


@pytest.fixture(scope="module")
def K():
    import kv_cache_compression_kvsculpt_b200 as K
    return K


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kvs_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(K):
    names = header_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(K.lib, n), n


def test_version(K):
    assert "sm_100a" in K.kvs_version()


def _cpu_batch(K, B=3, d=128, n_q=40, z=30, k=None):
    return K.KvsBatch.uniform(B, d, n_q, z, k, device="cpu")


def test_workspace_sizes(K):
    b = _cpu_batch(K, k=7)
    ws = K.kvs_workspace_bytes(b)
    assert ws > 4 * 3 * 40 * 30  # at least the score buffer
    assert ws % 256 == 0
    st = K.kvs_lbfgs_state_bytes(b, 10)
    assert st >= 4 * 3 * 7 * 128 * (4 + 2 * 11)
    assert K.kvs_lbfgs_state_bytes(b, 16) == 0   # history above 15 is rejected
    assert K.kvs_workspace_bytes(_cpu_batch(K, d=96)) == 0


def test_argument_errors_before_launch(K):
    lib = K.lib
    b = _cpu_batch(K, k=7)
    fake = ctypes.c_void_p(1 << 20)      # aligned, never dereferenced on error paths
    null = None
    big = 1 << 40
    # null workspace
    assert lib.kvs_targets(b.ref, fake, fake, fake, fake, fake, null, null, big, null) == -1
    # unaligned workspace
    assert lib.kvs_targets(b.ref, fake, fake, fake, fake, fake, null, ctypes.c_void_p(8), big,
                           null) == -1
    # too small a workspace
    assert lib.kvs_loss_grad(b.ref, fake, fake, fake, fake, fake, 1.0, 1.0, fake, null, null,
                             fake, 16, null) == -4
    # unsupported head dimension
    b96 = _cpu_batch(K, d=96, k=7)
    assert lib.kvs_loss_grad(b96.ref, fake, fake, fake, fake, fake, 1.0, 1.0, fake, null, null,
                             fake, big, null) == -3
    # k larger than the zone for top-k
    bk = _cpu_batch(K, z=30, k=31)
    assert lib.kvs_init_topk(bk.ref, fake, fake, fake, fake, null) == -1
    # bad schedule (history 0)
    sc = K.Schedule(history=0).struct()
    st = ctypes.c_void_p(1 << 24)
    assert lib.kvs_lbfgs_step(b.ref, ctypes.byref(sc), fake, fake, fake, fake, fake, st, big,
                              null, null, fake, big, null) == -1
    # decreasing offsets
    bad = K.KvsBatch(128, [0, 10, 5], [0, 4, 8], [0, 2, 4], device="cpu")
    assert lib.kvs_loss_grad(bad.ref, fake, fake, fake, fake, fake, 1.0, 1.0, fake, null, null,
                             fake, big, null) == -1
    # misaligned tensor pointer
    assert lib.kvs_loss_grad(b.ref, ctypes.c_void_p((1 << 20) + 4), fake, fake, fake, fake, 1.0,
                             1.0, fake, null, null, fake, big, null) == -1
    spec = K.QuerySpec(B=1, d=64, g=1, m_q=2, n_syn=2, N=16, rope_base=0.5).struct()
    assert lib.kvs_build_queries(ctypes.byref(spec), fake, fake, fake, fake, null) == -1


def test_pilot_allocate_golden(K, golden_dir):
    with open(os.path.join(golden_dir, "allocation_cases.json")) as fh:
        cases = json.load(fh)["cases"]
    for c in cases:
        got = K.kvs_pilot_allocate(c["mse"], c["total"], c["k_min"], c["k_max"], c["alpha"])
        assert got.tolist() == c["expect"], c["why"]


@pytest.mark.parametrize("seed", range(20))
def test_pilot_allocate_matches_oracle(K, seed):
    r = np.random.default_rng(500 + seed)
    B = int(r.integers(1, 60))
    k_min = int(r.integers(1, 20))
    k_max = r.integers(k_min, 2000, size=B).astype(np.int32)
    total = int(r.integers(B * k_min, int(k_max.sum()) + 1))
    mse = np.exp(r.uniform(-8, 4, size=B)).astype(np.float32)
    if seed % 5 == 0:
        mse[:: 3] = 0.0       # zero weights fall back to k_min
    got = K.kvs_pilot_allocate(mse, total, k_min, k_max, 0.5)
    want = O.pilot_allocate(mse.astype(np.float64), total, k_min, k_max, 0.5)
    assert got.tolist() == want.tolist()


def test_pilot_allocate_rejects_infeasible(K):
    with pytest.raises(K.KvsError):
        K.kvs_pilot_allocate([1.0, 2.0], 100, 16, [40, 40])
    with pytest.raises(K.KvsError):
        K.kvs_pilot_allocate([1.0, 2.0], 10, 16, [40, 40])


def test_lbfgs_state_layout(K):
    b = K.KvsBatch(128, [0, 40, 70], [0, 30, 60], [0, 7, 12], device="cpu")
    for h in (1, 3, 10, 15):
        L = K.kvs_lbfgs_state_layout(b, h)
        total = K.kvs_lbfgs_state_bytes(b, h)
        n = 12 * 128 * 4  # sum k_b * d floats
        assert L["slots"] == h + 1 and L["ring_stride"] == n
        assert L["scalar_bytes"] >= 16 and L["scalars"] + 2 * L["scalar_bytes"] <= L["x"]
        for f in ("off_f", "off_count", "off_head"):
            assert 0 <= L[f] <= L["scalar_bytes"] - 4 and L[f] % 4 == 0
        assert len({L["off_f"], L["off_count"], L["off_head"]}) == 3
        vecs = [L["x"], L["g"], L["dir"]]
        assert all(v % 256 == 0 for v in vecs + [L["ring_s"], L["ring_y"]])
        assert all(b1 - a >= n for a, b1 in zip(vecs, vecs[1:]))
        assert L["ring_s"] >= L["dir"] + n and L["ring_y"] >= L["ring_s"] + (h + 1) * n
        assert L["ring_y"] + (h + 1) * n <= total
    with pytest.raises(K.KvsError):
        K.kvs_lbfgs_state_layout(b, 16)
