"""Seeded synthetic inputs for the KVSculpt distillation solve.

This module is shared by the float64 oracle (``oracle/``) and by the CUDA
path's tests and benchmark.  It holds *no* arithmetic of the method: it only
draws random numbers and lays them out the way a transformer's KV cache would
hold them.  The one transformation it applies, the rotary position embedding of
keys and context queries, stands in for the model that produced the cache (the
method receives an already RoPE'd cache, KVSculpt page "Problem Statement":
after RoPE the pairs live in a continuous embedding space).  Everything the
method computes from these tensors (de-RoPE and re-embedding of synthetic
queries, targets, importance, fitting, L-BFGS, allocation) lives on each side
separately.

Workload shapes follow the paper's evaluation setting, Qwen2.5-1.5B-Instruct
with 2048-token contexts (KVSculpt page "Experimental Results"): 28 layers,
2 KV heads of dimension 128 and 6 query heads per KV head (GQA).  No model
weights or texts are used: every tensor is drawn from the distributions below.

* content keys  ~ N(0, 1), 4 outlier channels (per KV head, drawn without
  replacement) multiplied by 8, then by a per-layer key scale (1, or
  log-uniform in [0.5, 4] for the multi-layer workloads), RoPE'd at their
  context position 0..N-1 (rotate-half pairing, theta_i = base^(-2i/d));
* values        ~ N(0, 1), not rotated;
* query content ~ N(0, 1) per query head and context position; retain
  queries are RoPE'd at the retain-zone positions N-m..N-1; context queries
  for synthetic future queries are RoPE'd at n_syn positions drawn uniformly
  without replacement from [0, N) and sorted ascending (the draw is the
  method's own random choice, passed to both sides as an input).

Every problem (sequence, layer, KV head) draws from its own Philox stream keyed
by ``(seed, sequence, layer, head)``, so any subset of a batch can be
regenerated bit-identically on its own.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np

__all__ = [
    "Workload", "Batch", "WORKLOADS", "k_from_ratio", "generate", "make_batch",
    "subset", "restart_inits",
]


def k_from_ratio(r: float, z: int) -> int:
    """Compressed size for ratio r of a compress zone of z pairs (round half up)."""
    return int(math.floor(r * z + 0.5))


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape, distribution and schedule numbers of one synthetic workload."""
    name: str
    n_seq: int
    n_layers: int
    n_kv_heads: int
    d: int
    N: int
    m: int                 # retain zone size (newest pairs, kept verbatim)
    g: int                 # query heads per KV head (GQA group)
    n_syn: int             # synthetic future queries per query head
    k: int                 # uniform compressed size per problem
    layer_scale: bool      # per-layer key scale log-uniform in [0.5, 4]
    outer: int             # outer iterations (value re-fits)
    steps: int             # L-BFGS steps per outer iteration
    history: int = 10
    lam: float = 1e-3
    w_out: float = 1.0
    w_lse: float = 1.0
    rope_base: float = 1e6
    n_outlier: int = 4
    outlier_mult: float = 8.0
    adaptive: bool = False  # pilot run + budget reallocation before the solve
    pilot_outer: int = 12
    pilot_steps: int = 5
    k_min: int = 16
    alpha: float = 0.5

    @property
    def z(self) -> int:
        return self.N - self.m

    @property
    def m_q(self) -> int:
        return self.m

    @property
    def n_q(self) -> int:
        return self.g * (self.m_q + self.n_syn)

    @property
    def B(self) -> int:
        return self.n_seq * self.n_layers * self.n_kv_heads

    def problem_ids(self):
        return [(s, l, h) for s in range(self.n_seq) for l in range(self.n_layers)
                for h in range(self.n_kv_heads)]

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _qwen_cache(name, r, **kw):
    z = 2048 - 128
    return Workload(name=name, n_seq=1, n_layers=28, n_kv_heads=2, d=128, N=2048, m=128,
                    g=6, n_syn=512, k=k_from_ratio(r, z), layer_scale=True,
                    outer=40, steps=5, **kw)


WORKLOADS = {
    # one head-problem, d=64, N=256 (m=32) -> k=64, 32 retain + 96 synthetic queries
    "single_d64": Workload("single_d64", 1, 1, 1, d=64, N=256, m=32, g=1, n_syn=96, k=64,
                           layer_scale=False, outer=20, steps=5),
    # one Qwen2.5-1.5B-shaped layer: 2 KV heads x d=128, GQA 6, N=2048, m=128, r=0.5
    "qwen_layer": Workload("qwen_layer", 1, 1, 2, d=128, N=2048, m=128, g=6, n_syn=512,
                           k=k_from_ratio(0.5, 1920), layer_scale=False, outer=40, steps=5),
    # full 28-layer x 2-KV-head cache at r = 0.3 / 0.5 / 0.7
    "qwen_cache_r03": _qwen_cache("qwen_cache_r03", 0.3),
    "qwen_cache_r05": _qwen_cache("qwen_cache_r05", 0.5),
    "qwen_cache_r07": _qwen_cache("qwen_cache_r07", 0.7),
    # adaptive allocation at r = 0.5: 60-step pilot, then ragged k
    "qwen_cache_adaptive": _qwen_cache("qwen_cache_adaptive", 0.5, adaptive=True),
    # long context throughput mode: 8 sequences x 56 problems, N=8192, m=256, r=0.3
    "longctx": Workload("longctx", 8, 28, 2, d=128, N=8192, m=256, g=6, n_syn=1024,
                        k=k_from_ratio(0.3, 8192 - 256), layer_scale=True, outer=40, steps=5),
}


@dataclasses.dataclass
class Batch:
    """Host tensors of a batch of head-problems (float32 / int32 / int64).

    Rows are concatenated over problems; ``*_off`` hold the B+1 row offsets.
    """
    wl: Workload
    ids: list                 # (sequence, layer, head) per problem
    key_scale: np.ndarray     # [B] float64
    Kz: np.ndarray            # [sum z, d] RoPE'd keys of the compress zone (positions 0..z-1)
    Vz: np.ndarray            # [sum z, d]
    Kr: np.ndarray            # [B*m, d] retain-zone keys (positions z..N-1)
    Vr: np.ndarray            # [B*m, d]
    q_retain: np.ndarray      # [B*g*m_q, d] retain queries, RoPE'd at N-m_q..N-1, row (head, t)
    q_ctx: np.ndarray         # [B*g*n_syn, d] context queries RoPE'd at pos, row (head, j)
    pos: np.ndarray           # [B*g*n_syn] int32 sampled context positions, ascending per head
    z_off: np.ndarray         # [B+1] int64
    q_off: np.ndarray         # [B+1] int64 (training-query rows per problem = g*(m_q+n_syn))

    @property
    def B(self) -> int:
        return len(self.ids)

    def problem(self, b: int) -> dict:
        """Views of problem b's tensors."""
        wl = self.wl
        z0, z1 = self.z_off[b], self.z_off[b + 1]
        nr = wl.g * wl.m_q
        ns = wl.g * wl.n_syn
        return dict(
            Kz=self.Kz[z0:z1], Vz=self.Vz[z0:z1],
            Kr=self.Kr[b * wl.m:(b + 1) * wl.m], Vr=self.Vr[b * wl.m:(b + 1) * wl.m],
            q_retain=self.q_retain[b * nr:(b + 1) * nr],
            q_ctx=self.q_ctx[b * ns:(b + 1) * ns],
            pos=self.pos[b * ns:(b + 1) * ns],
        )


def _rope_model(x: np.ndarray, positions: np.ndarray, base: float) -> np.ndarray:
    """Rotary embedding as the model applies it (rotate-half pairing, float64)."""
    d = x.shape[-1]
    half = d // 2
    inv = base ** (-np.arange(half, dtype=np.float64) * 2.0 / d)
    ang = positions.astype(np.float64)[:, None] * inv[None, :]
    c, s = np.cos(ang), np.sin(ang)
    lo, hi = x[:, :half], x[:, half:]
    return np.concatenate([lo * c - hi * s, hi * c + lo * s], axis=1)


def _stream(seed: int, *key: int) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(np.random.SeedSequence([seed, *key])))


def layer_key_scale(wl: Workload, seed: int, layer: int) -> float:
    if not wl.layer_scale:
        return 1.0
    rng = _stream(seed, 1 << 20, layer)
    return float(math.exp(rng.uniform(math.log(0.5), math.log(4.0))))


def generate(wl: Workload, seed: int, seq: int, layer: int, head: int):
    """Draw one head-problem; returns float32/int32 numpy arrays."""
    rng = _stream(seed, seq, layer, head)
    d, N, m = wl.d, wl.N, wl.m
    scale = layer_key_scale(wl, seed, layer)
    kc = rng.standard_normal((N, d))
    outl = rng.choice(d, wl.n_outlier, replace=False)
    kc[:, outl] *= wl.outlier_mult
    kc *= scale
    K = _rope_model(kc, np.arange(N), wl.rope_base).astype(np.float32)
    V = rng.standard_normal((N, d)).astype(np.float32)
    qr, qc, ps = [], [], []
    t_ret = np.arange(N - wl.m_q, N)
    for _h in range(wl.g):
        c_ret = rng.standard_normal((wl.m_q, d))
        qr.append(_rope_model(c_ret, t_ret, wl.rope_base))
        p = np.sort(rng.choice(N, wl.n_syn, replace=False))
        c_ctx = rng.standard_normal((wl.n_syn, d))
        qc.append(_rope_model(c_ctx, p, wl.rope_base))
        ps.append(p)
    z = N - m
    return dict(
        Kz=K[:z], Vz=V[:z], Kr=K[z:], Vr=V[z:],
        q_retain=np.concatenate(qr).astype(np.float32),
        q_ctx=np.concatenate(qc).astype(np.float32),
        pos=np.concatenate(ps).astype(np.int32),
        key_scale=scale,
    )


def make_batch(wl: Workload, seed: int = 0, ids: Optional[Sequence] = None) -> Batch:
    """Generate the batch of problems ``ids`` (default: every problem of wl)."""
    ids = list(wl.problem_ids() if ids is None else ids)
    B, d, z = len(ids), wl.d, wl.z
    nr, ns = wl.g * wl.m_q, wl.g * wl.n_syn
    Kz = np.empty((B * z, d), np.float32)
    Vz = np.empty((B * z, d), np.float32)
    Kr = np.empty((B * wl.m, d), np.float32)
    Vr = np.empty((B * wl.m, d), np.float32)
    q_retain = np.empty((B * nr, d), np.float32)
    q_ctx = np.empty((B * ns, d), np.float32)
    pos = np.empty((B * ns,), np.int32)
    scales = np.empty((B,), np.float64)
    for b, (s, l, h) in enumerate(ids):
        p = generate(wl, seed, s, l, h)
        Kz[b * z:(b + 1) * z] = p["Kz"]
        Vz[b * z:(b + 1) * z] = p["Vz"]
        Kr[b * wl.m:(b + 1) * wl.m] = p["Kr"]
        Vr[b * wl.m:(b + 1) * wl.m] = p["Vr"]
        q_retain[b * nr:(b + 1) * nr] = p["q_retain"]
        q_ctx[b * ns:(b + 1) * ns] = p["q_ctx"]
        pos[b * ns:(b + 1) * ns] = p["pos"]
        scales[b] = p["key_scale"]
    z_off = np.arange(B + 1, dtype=np.int64) * z
    q_off = np.arange(B + 1, dtype=np.int64) * wl.n_q
    return Batch(wl, ids, scales, Kz, Vz, Kr, Vr, q_retain, q_ctx, pos, z_off, q_off)


def subset(wl: Workload, count: int, seed: int = 0) -> list:
    """A fixed, seeded choice of ``count`` problem ids of wl (sorted)."""
    allids = wl.problem_ids()
    rng = _stream(seed, 7 << 20)
    pick = np.sort(rng.choice(len(allids), min(count, len(allids)), replace=False))
    return [allids[i] for i in pick]


def restart_inits(z_counts: Sequence[int], k_counts: Sequence[int], restarts: int,
                  seed: int = 0) -> np.ndarray:
    """Initial key subsets of a random-restart search: for restart r and problem b,
    k_b distinct zone positions drawn uniformly without replacement from
    [0, z_b), sorted ascending.  Returns int32 [restarts, sum k_b] (problem b's
    entries at its c_off[b] ..).  The draw is the search's own random choice,
    passed to both sides as an input; each (restart, problem) has its own stream."""
    z_counts = [int(z) for z in z_counts]
    k_counts = [int(k) for k in k_counts]
    if len(z_counts) != len(k_counts) or any(not 1 <= k <= z for k, z in zip(k_counts, z_counts)):
        raise ValueError("each problem needs 1 <= k_b <= z_b")
    out = np.empty((restarts, sum(k_counts)), np.int32)
    for r in range(restarts):
        c = 0
        for b, (z, k) in enumerate(zip(z_counts, k_counts)):
            rng = _stream(seed, 9 << 20, r, b)
            out[r, c:c + k] = np.sort(rng.choice(z, k, replace=False))
            c += k
    return out
