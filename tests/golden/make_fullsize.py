"""Write fullsize_oracle.json: the float64 oracle's results on seeded subsets
of the full-size workloads (every value comes from ``oracle/`` alone).

The GPU parity tests compare kvs_compress_batch (and the adaptive path) on the
same problems with these stored results, because the oracle needs minutes per
problem at these sizes.  Cases:

* the 28-layer x 2-KV-head cache at r = 0.3, 0.5 and 0.7 ("KVSculpt: KV Cache
  Compression as Distillation", summary section 4 "Experimental Results"):
  three problems each -- the layers with the largest and the smallest
  per-layer key scale, and one in between -- through the whole 40 x 5
  schedule;
* adaptive allocation at r = 0.5 (summary section 2 "Adaptive Budget
  Allocation") on four problems: a 12 x 5 pilot at uniform k, the allocation
  by pilot output MSE, then the full solve at the allocated sizes;
* one long-context head-problem (N = 8192, m = 256, r = 0.3) through the whole
  40 x 5 schedule.

Inputs are the training queries built by the oracle and rounded to float32
(the same float32 tensors the GPU tests feed to the library), plus the
workload's float32 zone keys and values.  Checksums of those inputs are stored
so that a test can tell when the generator has changed.

Each solve is also repeated with loss and gradient evaluations perturbed at the
relative precision of the library's arithmetic (oracle.perturb, two seeds), and
once with the library's own rounding emulated in float64 (oracle.perturb
emulated_evaluations): the final losses of those runs ("band", "emulated")
show how far a run of that precision can legitimately end from the exact one
on this (non-convex, fixed-length) trajectory.  The adaptive case's runs are
taken at the oracle's allocation.

Run:  python tests/golden/make_fullsize.py   (about 2 hours on 8 cores)
      python tests/golden/make_fullsize.py --add-emulated   (only the emulated
      runs, added to an existing file)
"""
from __future__ import annotations

import json
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle as O  # noqa: E402
import workload as W  # noqa: E402
from oracle.perturb import GPU_LEVELS, emulated_evaluations, noisy_evaluations  # noqa: E402

BAND_SEEDS = 2

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "fullsize_oracle.json")

# (sequence, layer, KV head): layer 21 has the largest key scale of the seeded
# cache (3.97), layer 22 the smallest (0.54), layer 13 lies in between (1.14)
CACHE_IDS = [(0, 21, 0), (0, 22, 1), (0, 13, 1)]
ADAPTIVE_IDS = [(0, 21, 0), (0, 22, 1), (0, 2, 0), (0, 17, 1)]
LONGCTX_IDS = [(0, 21, 0)]


def float32_inputs(wl, ids):
    """Per problem: oracle training queries rounded to float32, zone keys and values."""
    bt = W.make_batch(wl, 0, ids)
    out = []
    for b in range(bt.B):
        p = bt.problem(b)
        Q = O.build_queries(p["q_retain"], p["q_ctx"], p["pos"], wl.g, wl.m_q, wl.n_syn, wl.N,
                            wl.rope_base).astype(np.float32)
        out.append((Q, p["Kz"], p["Vz"]))
    return out


def checksum(x):
    x = np.asarray(x, np.float64)
    return [float(np.abs(x).sum()), float((x * x).sum())]


def schedule(wl, pilot=False):
    return O.Schedule(outer=wl.pilot_outer if pilot else wl.outer,
                      steps=wl.pilot_steps if pilot else wl.steps, history=wl.history,
                      lam=wl.lam, w_out=wl.w_out, w_lse=wl.w_lse)


def result_record(r):
    return {"trace": [float(v) for v in r["trace"]], "loss": float(r["loss"]),
            "mse_out": float(r["mse_out"]), "mse_lse": float(r["mse_lse"]),
            "status": int(r["status"]), "trials": int(r["trials"])}


def band(Q, Kz, Vz, k, sched):
    """Final losses of the schedule with perturbed evaluations (oracle.perturb)."""
    return [float(O.compress(Q, Kz, Vz, k, sched, evaluate=noisy_evaluations(*GPU_LEVELS, s))
                  ["loss"]) for s in range(BAND_SEEDS)]


def emulated(Q, Kz, Vz, k, sched):
    """Final loss of the schedule with the library's rounding emulated."""
    return float(O.compress(Q, Kz, Vz, k, sched, evaluate=emulated_evaluations())["loss"])


def uniform_case(name, ids):
    wl = W.WORKLOADS[name]
    t0 = time.time()
    probs = []
    for (Q, Kz, Vz), pid in zip(float32_inputs(wl, ids), ids):
        r = O.compress(Q, Kz, Vz, wl.k, schedule(wl))
        rec = result_record(r)
        rec["band"] = band(Q, Kz, Vz, wl.k, schedule(wl))
        rec["emulated"] = emulated(Q, Kz, Vz, wl.k, schedule(wl))
        rec.update(id=list(pid), k=wl.k, checksum_Q=checksum(Q), checksum_Kz=checksum(Kz),
                   checksum_Vz=checksum(Vz))
        probs.append(rec)
        print(f"{name} {pid}: loss {rec['loss']:.6g} ({time.time() - t0:.0f} s)", flush=True)
    return {"workload": name, "problems": probs}


def adaptive_case(ids):
    wl = W.WORKLOADS["qwen_cache_adaptive"]
    inp = float32_inputs(wl, ids)
    total = wl.k * len(ids)
    t0 = time.time()
    res = O.adaptive_compress([dict(Q=Q, Kz=Kz, Vz=Vz) for Q, Kz, Vz in inp], total,
                              schedule(wl), schedule(wl, pilot=True), wl.k_min, wl.alpha)
    probs = []
    for b, (pid, (Q, Kz, Vz)) in enumerate(zip(ids, inp)):
        rec = result_record(res["results"][b])
        rec["band"] = band(Q, Kz, Vz, int(res["k"][b]), schedule(wl))
        rec["emulated"] = emulated(Q, Kz, Vz, int(res["k"][b]), schedule(wl))
        rec.update(id=list(pid), k=int(res["k"][b]), pilot_mse=float(res["pilot_mse"][b]),
                   checksum_Q=checksum(Q), checksum_Kz=checksum(Kz), checksum_Vz=checksum(Vz))
        probs.append(rec)
    print(f"adaptive: k {list(res['k'])} ({time.time() - t0:.0f} s)", flush=True)
    return {"workload": wl.name, "total": int(total), "problems": probs}


def add_emulated():
    """Add the emulated-rounding run to every problem of an existing file."""
    with open(OUT) as fh:
        out = json.load(fh)
    for name, case in out["cases"].items():
        wl = W.WORKLOADS[name]
        ids = [tuple(p["id"]) for p in case["problems"]]
        for (Q, Kz, Vz), p in zip(float32_inputs(wl, ids), case["problems"]):
            if "emulated" in p:
                continue
            t0 = time.time()
            p["emulated"] = emulated(Q, Kz, Vz, int(p["k"]), schedule(wl))
            print(f"{name} {p['id']}: emulated {p['emulated'] / p['loss']:.4f}x "
                  f"({time.time() - t0:.0f} s)", flush=True)
            with open(OUT, "w") as fh:
                json.dump(out, fh, indent=1)


def add_pilot_bands():
    """Add, for every adaptive problem, the pilot MSE of the pilot schedule run with
    perturbed evaluations (the same levels and seeds as the final-loss bands) and
    with the library's rounding emulated: the pilot is as trajectory-sensitive as
    the full solve, so its MSE is compared with a band too."""
    with open(OUT) as fh:
        out = json.load(fh)
    case = out["cases"]["qwen_cache_adaptive"]
    wl = W.WORKLOADS["qwen_cache_adaptive"]
    ids = [tuple(p["id"]) for p in case["problems"]]
    k_uni = case["total"] // len(ids)
    pilot = schedule(wl, pilot=True)
    for (Q, Kz, Vz), p in zip(float32_inputs(wl, ids), case["problems"]):
        if "pilot_band" in p:
            continue
        t0 = time.time()
        p["pilot_band"] = [float(O.compress(Q, Kz, Vz, k_uni, pilot,
                                            evaluate=noisy_evaluations(*GPU_LEVELS, s))["mse_out"])
                           for s in range(BAND_SEEDS)]
        p["pilot_emulated"] = float(O.compress(Q, Kz, Vz, k_uni, pilot,
                                               evaluate=emulated_evaluations())["mse_out"])
        print(f"adaptive {p['id']}: pilot band {[round(x / p['pilot_mse'], 4) for x in p['pilot_band']]}"
              f" emulated {p['pilot_emulated'] / p['pilot_mse']:.4f} ({time.time() - t0:.0f} s)",
              flush=True)
        with open(OUT, "w") as fh:
            json.dump(out, fh, indent=1)


def main():
    if "--add-emulated" in sys.argv:
        return add_emulated()
    if "--add-pilot-bands" in sys.argv:
        return add_pilot_bands()
    out = {"generator": "tests/golden/make_fullsize.py (oracle/ only)", "seed": 0,
           "band_levels": list(GPU_LEVELS), "cases": {}}
    for name in ("qwen_cache_r03", "qwen_cache_r05", "qwen_cache_r07"):
        out["cases"][name] = uniform_case(name, CACHE_IDS)
    out["cases"]["qwen_cache_adaptive"] = adaptive_case(ADAPTIVE_IDS)
    out["cases"]["longctx"] = uniform_case("longctx", LONGCTX_IDS)
    with open(OUT, "w") as fh:
        json.dump(out, fh, indent=1)
    print("wrote", OUT)


if __name__ == "__main__":
    main()
