#!/usr/bin/env python
"""Throughput of the KVSculpt distillation solve on B200.

One step = the whole hot path over one batch of head-problems: training-query
construction, targets and importance, top-k keys, the initial ridge fit, then
`outer` x (`steps` L-BFGS steps + ridge re-fit), for every problem of the
workload (default: 28 layers x 2 KV heads of a Qwen2.5-1.5B-shaped cache,
N = 2048, m = 128, r = 0.5, 40 x 5 schedule).  Inputs are resident in HBM when
the device-timed region starts; the e2e figure repeats the step through the
same C-ABI calls with the inputs copied from pinned host memory and the
compressed pairs copied back inside the timed region.

Prints one JSON line (rank 0).  `--impl reference` times the float64 CPU
oracle on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workload as W  # noqa: E402

METRIC = "head-problems compressed/sec at N=2048,r=0.5"  # the default workload's metric


def metric_for(wl: W.Workload) -> str:
    """The throughput metric of a workload, labelled with its context length and ratio."""
    r = round(wl.k / wl.z, 2)
    label = f"head-problems compressed/sec at N={wl.N},r={r:g}"
    return label + (" (adaptive allocation)" if wl.adaptive else "")


FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# CUDA-core fp32 FMA peak from unit counts and clock: 148 SMs x 128 lanes x 2 flop x 1.965 GHz
DERIVED_PEAKS = {"fp32_simt_tflops": 148 * 128 * 2 * 1.965e9 / 1e12}


# Sources of the loss/gradient kernels: the DRAM traffic recorded under profiles/
# holds only while these files are unchanged.
TRAFFIC_SOURCES = ["kvs_attn_fwd.cu", "kvs_attn_bwd.cu", "kvs_attn_tc.cuh", "kvs_tc.cuh"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "loss_grad_traffic_qwen_cache_r05.md")


def kernel_source_hash():
    h = hashlib.sha256()
    for f in TRAFFIC_SOURCES:
        with open(os.path.join(ROOT, "kv_cache_compression_kvsculpt_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def recorded_traffic(workload):
    """DRAM bytes of one loss/gradient evaluation (forward + key gradient) from the
    committed ncu summary, or None when the summary is missing, is for another
    workload, or predates the current kernel sources."""
    try:
        with open(TRAFFIC_FILE) as fh:
            kv = dict(line.strip("- \n").split(": ", 1) for line in fh if ": " in line)
    except OSError:
        return None
    if kv.get("workload") != workload or kv.get("source_sha256") != kernel_source_hash():
        return None
    try:
        return int(kv["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def describe(wl: W.Workload):
    return (f"{wl.name}: {wl.B} head-problems ({wl.n_seq} seq x {wl.n_layers} layers x "
            f"{wl.n_kv_heads} KV heads), d={wl.d}, N={wl.N}, m={wl.m}, z={wl.z}, k={wl.k}, "
            f"n_q={wl.g}x({wl.m_q}+{wl.n_syn})={wl.n_q}, schedule {wl.outer}x{wl.steps} L-BFGS, "
            f"history {wl.history}, lambda {wl.lam}")


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.rows = []
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([x.strip() for x in line.split(",")])

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm = [float(r[1]) for r in self.rows if len(r) > 8 and r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if len(r) > 8 and r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in self.rows:
            if len(r) > 8:
                for n, v in zip(names, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(self.rows)}


# ---------------------------------------------------------------- GPU arm

def group_size(group):
    import torch.distributed as dist
    return dist.get_world_size(group)


class Job:
    """Device buffers of one rank's batch and the calls of one step."""

    def __init__(self, wl, seqs, dev, group=None, problems=None):
        import torch
        import kv_cache_compression_kvsculpt_b200 as K
        self.K, self.torch, self.wl, self.group = K, torch, wl, group
        ids = [(s, l, h) for s in seqs for l in range(wl.n_layers) for h in range(wl.n_kv_heads)]
        if problems:
            ids = ids[:problems]  # a reduced batch (kernel profiling)
        self.bt = W.make_batch(wl, 0, ids)
        B = self.bt.B
        self.host = {
            "q_retain": torch.from_numpy(self.bt.q_retain).pin_memory(),
            "q_ctx": torch.from_numpy(self.bt.q_ctx).pin_memory(),
            "pos": torch.from_numpy(self.bt.pos).pin_memory(),
            "Kz": torch.from_numpy(self.bt.Kz).pin_memory(),
            "Vz": torch.from_numpy(self.bt.Vz).pin_memory(),
        }
        self.dev = {k: v.to(dev) for k, v in self.host.items()}
        self.batch = K.KvsBatch(wl.d, self.bt.q_off, self.bt.z_off,
                                np.arange(B + 1, dtype=np.int64) * wl.k)
        self.spec = K.QuerySpec(B, wl.d, wl.g, wl.m_q, wl.n_syn, wl.N, wl.rope_base)
        self.sched = K.Schedule(outer=wl.outer, steps=wl.steps, history=wl.history, lam=wl.lam,
                                w_out=wl.w_out, w_lse=wl.w_lse)
        self.pilot = K.Schedule(outer=wl.pilot_outer, steps=wl.pilot_steps, history=wl.history,
                                lam=wl.lam, w_out=wl.w_out, w_lse=wl.w_lse)
        self.Q = torch.empty((self.batch.sum_q, wl.d), device=dev)
        self.Kc = torch.empty((self.batch.sum_c, wl.d), device=dev)
        self.Vc = torch.empty_like(self.Kc)
        self.trace = torch.empty((B, wl.outer + 1), device=dev)
        self.parts = torch.empty((B, 2), device=dev)
        self.status = torch.empty(B, dtype=torch.int32, device=dev)
        self.ws = K.alloc_workspace(self.batch, device=dev)
        self.state = K.alloc_state(self.batch, wl.history, device=dev)
        self.total = wl.k * B * (1 if group is None else group_size(group))
        self.out_host = {"Kc": torch.empty(self.Kc.shape).pin_memory(),
                         "Vc": torch.empty(self.Vc.shape).pin_memory()}

    def step(self, d=None):
        K = self.K
        d = d or self.dev
        K.kvs_build_queries(self.spec, d["q_retain"], d["q_ctx"], d["pos"], self.Q)
        if self.wl.adaptive:
            # pilot at uniform k, pooled allocation (one all-gather over ranks), full solve
            from kv_cache_compression_kvsculpt_b200 import adaptive
            r = adaptive.compress_adaptive(self.wl.d, self.bt.q_off, self.bt.z_off, self.Q,
                                           d["Kz"], d["Vz"], self.total, self.sched, self.pilot,
                                           group=self.group)
            self.Kc, self.Vc, self.trace, self.parts, self.status = (
                r["Kc"], r["Vc"], r["trace"], r["parts"], r["status"])
            self.batch = K.KvsBatch(self.wl.d, self.bt.q_off, self.bt.z_off, r["c_off"])
            self.k_alloc = r["k"]
            return
        K.kvs_compress_batch(self.batch, self.sched, self.Q, d["Kz"], d["Vz"], self.Kc, self.Vc,
                             None, self.trace, self.parts, self.status, self.state, self.ws)

    def step_e2e(self):
        """Same step from pinned host inputs, compressed pairs copied back."""
        d = {k: self.dev[k].copy_(v, non_blocking=True) for k, v in self.host.items()}
        self.step(d)
        self.out_host["Kc"].copy_(self.Kc, non_blocking=True)
        self.out_host["Vc"].copy_(self.Vc, non_blocking=True)

    def h2d_bytes(self):
        return sum(v.numel() * v.element_size() for v in self.host.values())

    def d2h_bytes(self):
        return sum(v.numel() * v.element_size() for v in self.out_host.values())


def rank_sequences(wl, rank, world):
    """Sequences (each n_layers x n_kv_heads head-problems) this rank compresses.
    A workload of several sequences is partitioned over the ranks (the total is
    fixed: strong scaling; the rank count must divide it); a one-sequence
    workload gives every rank a sequence of its own (weak scaling)."""
    if wl.n_seq > 1:
        if wl.n_seq % world:
            raise SystemExit(f"{wl.name}: {wl.n_seq} sequences do not split over {world} ranks")
        return list(range(rank, wl.n_seq, world)), "strong"
    return [rank], "weak"


def time_region(torch, fn, n, dist=None):
    """Device time (ms) of n calls of fn on the current stream, max over ranks."""
    st = torch.cuda.current_stream()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(n):
        fn()
    e1.record(st)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    if dist:
        t = torch.tensor([ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
        dist.barrier()
    return ms


def loss_grad_roofline(job, peaks, reps=20):
    """Time kvs_loss_grad (the dominant evaluation) over the batch at the solved point."""
    torch, K, wl = job.torch, job.K, job.wl
    B = job.batch.B
    # the solve's workspace when it is large enough for the batch's (possibly
    # allocated) k, else one of that size
    ws = (job.ws if K.kvs_workspace_bytes(job.batch) <= job.ws.numel()
          else K.alloc_workspace(job.batch))
    Y = torch.empty_like(job.Q)
    lse = torch.empty(job.batch.sum_q, device=job.Q.device)
    K.kvs_targets(job.batch, job.Q, job.dev["Kz"], job.dev["Vz"], Y, lse, None, ws)
    loss = torch.empty(B, device=job.Q.device)
    dK = torch.empty_like(job.Kc)

    def ev():
        K.kvs_loss_grad(job.batch, job.Q, job.Kc, job.Vc, Y, lse, 1.0, 1.0, loss, None, dK, ws)

    for _ in range(3):
        ev()
    ms = time_region(torch, ev, reps) / reps
    flops = 8.0 * wl.n_q * wl.k * wl.d * B
    achieved = flops / (ms * 1e-3) / 1e12
    return ms, flops, achieved


def run_loss_grad_only(args, job, wl, rank, world, dist):
    """The dominant evaluation alone: kvs_loss_grad over the batch at its Select+Fit
    point (one solve with no outer iterations first), `--steps` timed calls after
    `--warmup` untimed ones.  A kernel-level measurement, not the bench step."""
    torch, K = job.torch, job.K
    job.sched.outer = 0
    job.step()
    B = job.batch.B
    Y = torch.empty_like(job.Q)
    lse = torch.empty(job.batch.sum_q, device=job.Q.device)
    K.kvs_targets(job.batch, job.Q, job.dev["Kz"], job.dev["Vz"], Y, lse, None, job.ws)
    loss = torch.empty(B, device=job.Q.device)
    dK = torch.empty_like(job.Kc)

    def ev():
        K.kvs_loss_grad(job.batch, job.Q, job.Kc, job.Vc, Y, lse, 1.0, 1.0, loss, None, dK, job.ws)

    for _ in range(args.warmup):
        ev()
    ms = time_region(torch, ev, args.steps, dist) / args.steps
    # each call on its own, with the finiteness of its results (a kernel whose
    # bounded wait gave up returns NaN)
    per, bad = [], 0
    for _ in range(args.steps):
        per.append(time_region(torch, ev, 1, dist))
        bad += int(not (torch.isfinite(loss).all() and torch.isfinite(dK).all()))
    flops = 8.0 * wl.n_q * wl.k * wl.d * B
    peaks, peak_src = load_peaks()
    peak = peaks.get(args.peak_key, FALLBACK_PEAKS.get(args.peak_key))
    if rank == 0:
        print(json.dumps({"metric": "kvs_loss_grad ms per call (whole batch)", "value": round(ms, 4),
                          "unit": "ms", "problems": B, "workload": wl.name,
                          "achieved_tflops": round(flops / (ms * 1e-3) / 1e12, 2),
                          "frac": round(flops / (ms * 1e-3) / 1e12 / peak, 4),
                          "per_call_ms": {"min": round(min(per), 4), "median":
                                          round(statistics.median(per), 4),
                                          "max": round(max(per), 4)},
                          "calls_with_nan": bad,
                          "peak_source": f"{peak_src} {args.peak_key}"}), flush=True)


def run_fit_only(args, job, wl, rank, world, dist):
    """The ridge fit alone: kvs_fit_values over the batch at its Select+Fit point
    (one solve with no outer iterations first), `--steps` timed calls after
    `--warmup` untimed ones.  A kernel-level measurement, not the bench step."""
    torch, K = job.torch, job.K
    job.sched.outer = 0
    job.step()
    B = job.batch.B
    Y = torch.empty_like(job.Q)
    lse = torch.empty(job.batch.sum_q, device=job.Q.device)
    K.kvs_targets(job.batch, job.Q, job.dev["Kz"], job.dev["Vz"], Y, lse, None, job.ws)
    Vc = torch.empty_like(job.Vc)
    status = torch.zeros(B, dtype=torch.int32, device=job.Q.device)

    def fit():
        K.kvs_fit_values(job.batch, job.Q, job.Kc, Y, wl.lam, Vc, status, job.ws)

    for _ in range(args.warmup):
        fit()
    ms = time_region(torch, fit, args.steps, dist) / args.steps
    if rank == 0:
        print(json.dumps({"metric": "kvs_fit_values ms per call (whole batch)", "value": round(ms, 4),
                          "unit": "ms", "problems": B, "workload": wl.name,
                          "status_nonzero": int((status != 0).sum())}), flush=True)


def run_gpu(args):
    import torch
    import kv_cache_compression_kvsculpt_b200 as K
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist_mod
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        dist = dist_mod
    torch.cuda.set_device(local)
    wl = W.WORKLOADS[args.workload]
    if args.outer is not None:
        wl = wl.with_(outer=args.outer)
    seqs, scaling = rank_sequences(wl, rank, world)
    job = Job(wl, seqs, dev="cuda", group=dist.group.WORLD if dist else None,
              problems=args.problems)
    if args.loss_grad_only:
        return run_loss_grad_only(args, job, wl, rank, world, dist)
    if args.fit_only:
        return run_fit_only(args, job, wl, rank, world, dist)
    for _ in range(args.warmup):
        job.step()
    torch.cuda.synchronize()
    st = int(torch.cuda.current_device())
    n0 = K.kvs_launch_count()
    with ClockSampler(st) as clk:
        ms = time_region(torch, job.step, args.steps, dist)
    launches = K.kvs_launch_count() - n0
    status = job.status.cpu().numpy()
    ms_step = ms / args.steps
    problems = job.batch.B * world  # every rank holds the same number of problems
    value = problems / (ms_step * 1e-3)
    # e2e through host buffers
    job.step_e2e()
    ms_e2e = time_region(torch, job.step_e2e, args.steps, dist) / args.steps
    e2e_value = problems / (ms_e2e * 1e-3)
    peaks, peak_src = load_peaks()
    lg_ms, lg_flops, lg_tflops = loss_grad_roofline(job, peaks)
    if args.peak_key in DERIVED_PEAKS:
        peak, peak_src = DERIVED_PEAKS[args.peak_key], "derived"
    else:
        peak = peaks.get(args.peak_key, FALLBACK_PEAKS.get(args.peak_key))
    final = job.trace[:, -1].cpu().numpy()
    first = job.trace[:, 0].cpu().numpy()
    out = {
        "metric": metric_for(wl),
        "value": round(value, 4),
        "unit": "head-problems/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 3),
        "higher_is_better": True,
        "scaling": scaling,
        "vs_baseline": None,
        "dtype": args.dtype_label,
        "data": "synthetic (seeded generator; stands in for Qwen2.5-1.5B-Instruct KV caches)",
        "config": {"workload": describe(wl), "problems_per_gpu": job.batch.B,
                   "l2": "inputs and per-step working set larger than L2 (126 MB)",
                   "parallelism": f"problem-sharded x{world}, no collective"},
        "e2e": {"value": round(e2e_value, 4), "unit": "head-problems/s",
                "h2d_bytes_per_step": job.h2d_bytes(), "d2h_bytes_per_step": job.d2h_bytes()},
        "loss_grad_evals_per_s": round(job.batch.B / (lg_ms * 1e-3), 1),  # per rank's batch
        "roofline": {"kernel": "kvs_loss_grad (forward + dKc backward, whole batch)",
                     "bound": args.bound, "achieved": round(lg_tflops, 3), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(lg_tflops / peak, 4),
                     "traffic": recorded_traffic(wl.name),
                     "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum of "
                                       "k_attn_fwd LOSS + k_attn_bwd DK, one launch each",
                     "peak_source": f"{peak_src} {args.peak_key}",
                     "ms_per_launch": round(lg_ms, 4),
                     "algorithmic_flops_per_launch": lg_flops},
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
        "quality": {"select_fit_loss_mean": float(np.mean(first)),
                    "final_loss_mean": float(np.mean(final)),
                    "status_nonzero": int((status != 0).sum())},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:  # the oracle beside one GPU only
        out["cpu_baseline"] = cpu_baseline(wl, budget_s=args.cpu_budget)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


# ---------------------------------------------------------------- oracle

class OracleRun:
    """The oracle's schedule on one problem of the workload: the set-up (query
    build, targets, top-k, first fit) once, then outer iterations one at a time."""

    def __init__(self, wl, pid=(0, 0, 0)):
        import oracle as O
        self.O, self.wl, self.pid = O, wl, pid
        t0 = time.perf_counter()
        bt = W.make_batch(wl, 0, [pid])
        p = bt.problem(0)
        Q = O.build_queries(p["q_retain"], p["q_ctx"], p["pos"], wl.g, wl.m_q, wl.n_syn, wl.N,
                            wl.rope_base)
        Y, lse = O.targets(Q, p["Kz"], p["Vz"])
        idx = O.topk_select(O.importance(Q, p["Kz"], lse), wl.k)
        Kc = np.asarray(p["Kz"], np.float64)[idx]
        self.Vc, _ = O.ridge_fit(Q, Kc, Y, wl.lam)
        f, g, _ = O.loss_grad(Q, Kc, self.Vc, Y, lse)
        self.st = O.LBFGSState(x=Kc.ravel().copy(), f=f, g=g.ravel())
        self.Q, self.Y, self.lse = Q, Y, lse
        self.t_setup = time.perf_counter() - t0

    def outer(self):
        """One outer iteration (steps L-BFGS steps, value re-fit); returns its seconds."""
        O, wl, d = self.O, self.wl, self.wl.d
        Q, Y, lse, Vc, st = self.Q, self.Y, self.lse, self.Vc, self.st
        t0 = time.perf_counter()
        fl = lambda x: O.loss_only(Q, x.reshape(-1, d), Vc, Y, lse)
        fg = lambda x: O.loss_grad(Q, x.reshape(-1, d), Vc, Y, lse)[1].ravel()
        for _ in range(wl.steps):
            O.lbfgs_step(st, fl, fg, wl.history)
        self.Vc, _ = O.ridge_fit(Q, st.x.reshape(-1, d), Y, wl.lam)
        f, g, _ = O.loss_grad(Q, st.x.reshape(-1, d), self.Vc, Y, lse)
        st.f, st.g = f, g.ravel()
        return time.perf_counter() - t0

    def per_problem(self, t_outer):
        """Seconds per head-problem of the whole schedule from the measured set-up and
        mean outer-iteration time (plus the pilot run of an adaptive workload)."""
        wl = self.wl
        total = self.t_setup + t_outer * wl.outer
        if wl.adaptive:
            total += self.t_setup + t_outer * wl.pilot_outer * wl.pilot_steps / wl.steps
        return total

    def describe(self, n_outer, threads):
        wl = self.wl
        s = (f"1 problem {self.pid} of {wl.name} on {threads} thread(s): query build, targets, "
             f"top-k and first fit timed once, then {n_outer} of the {wl.outer} outer "
             f"iterations ({wl.steps} L-BFGS steps + re-fit each) timed; per-problem time "
             f"extrapolated to the full schedule")
        if wl.adaptive:
            s += f", plus a {wl.pilot_outer}x{wl.pilot_steps} pilot extrapolated the same way"
        return s


def _cores():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def cpu_baseline(wl, budget_s=20.0):
    """The oracle as it stands on the host's cores (BLAS threads = all cores), outer
    iterations until budget_s, and one outer iteration on a single thread."""
    run = OracleRun(wl)
    times = [run.outer()]
    while len(times) < wl.outer and sum(times) < budget_s:
        times.append(run.outer())
    t = run.per_problem(float(np.mean(times)))
    out = {"value": round(1.0 / t, 6), "unit": "head-problems/s", "cores": _cores(),
           "kind": "oracle", "extrapolated": True, "sample": run.describe(len(times), _cores()),
           "seconds_per_problem": round(t, 2)}
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            one = OracleRun(wl)
            t1 = one.per_problem(one.outer())
        out["single_thread"] = {"value": round(1.0 / t1, 6), "unit": "head-problems/s",
                                "cores": 1, "seconds_per_problem": round(t1, 1),
                                "sample": one.describe(1, 1)}
    except ImportError:
        pass
    return out


def run_reference(args):
    """The oracle timed on the host cores.  One step = one outer iteration of the
    schedule on one problem (a bounded sample); the value extrapolates the measured
    set-up and outer-iteration times to whole head-problems per second."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = W.WORKLOADS[args.workload]
    if args.outer is not None:
        wl = wl.with_(outer=args.outer)
    run = OracleRun(wl)
    for _ in range(args.warmup):
        run.outer()
    times = [run.outer() for _ in range(args.steps)]
    per = run.per_problem(float(np.mean(times)))
    value = 1.0 / per
    sample = run.describe(args.steps, _cores())
    out = {"impl": "reference", "metric": metric_for(wl), "value": round(value, 6),
           "unit": "head-problems/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
           "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": round(float(np.mean(times)) * 1e3, 1),
           "step": "one outer iteration of one problem's schedule (value: whole problems/s, "
                   "extrapolated)",
           "extrapolated": True, "seconds_per_problem": round(per, 2),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic (seeded generator)", "config": {"workload": describe(wl)},
           "cpu_baseline": {"value": round(value, 6), "unit": "head-problems/s",
                            "cores": _cores(), "kind": "oracle", "sample": sample,
                            "extrapolated": True},
           "e2e": {"value": round(value, 6), "unit": "head-problems/s",
                   "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


# ---------------------------------------------------------------- ranks

def rank_env(base_env, world, rank, port):
    """Environment of rank `rank` of `world` processes on this node (one GPU each)."""
    env = dict(base_env)
    env.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
               LOCAL_WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    return env


def free_port():
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def spawn_ranks(world, argv, timeout_s=3600):
    """Run this script as `world` processes (rank 0 prints the JSON line); returns the
    first non-zero exit code, or 0.  A rank that fails ends the others."""
    port = free_port()
    procs = [subprocess.Popen([sys.executable, os.path.abspath(__file__), *argv],
                              env=rank_env(os.environ, world, r, port))
             for r in range(world)]
    rc = 0
    t_end = time.time() + timeout_s
    while procs:
        for p in list(procs):
            code = p.poll()
            if code is None:
                continue
            procs.remove(p)
            if code != 0 and rc == 0:
                rc = code
                t_end = min(t_end, time.time() + 60)  # give the others a minute
        if time.time() > t_end:
            for p in procs:
                p.kill()
            rc = rc or 124
            break
        time.sleep(0.2)
    return rc


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="qwen_cache_r05", choices=sorted(W.WORKLOADS))
    ap.add_argument("--outer", type=int, default=None, help="override the outer iterations")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--problems", type=int, default=None,
                    help="only the first N problems of the workload (kernel profiling)")
    ap.add_argument("--fit-only", action="store_true",
                    help="time kvs_fit_values alone over the batch (kernel-level)")
    ap.add_argument("--loss-grad-only", action="store_true",
                    help="time kvs_loss_grad alone (kernel measurement, not the bench step)")
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--bound", default="tensor")
    ap.add_argument("--peak-key", default="bf16_tflops")
    ap.add_argument("--dtype-label", default="bf16x3-f32acc")
    args = ap.parse_args()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU, launched here (torchrun sets WORLD_SIZE itself)
        sys.exit(spawn_ranks(args.gpus, sys.argv[1:]))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.gpus != world:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
