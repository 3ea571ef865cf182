"""Host logic of bench.py (CPU): the reference arm's JSON line, the work each rank
takes, and the guard that reports recorded DRAM traffic only for the kernel
sources it was measured on."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import workload as W  # noqa: E402


def test_reference_line_contract():
    # the float64 oracle on the smallest workload, one bounded sample
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "single_d64", "--steps", "1", "--warmup", "0",
                        "--cpu-budget", "2"], capture_output=True, text=True, timeout=600,
                       cwd=ROOT)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == "head-problems/s"
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["warmup"] == 0 and d["n_gpus"] == 1
    assert d["dtype"] == "f64" and d["vs_baseline"] is None
    assert d["config"]["workload"].startswith("single_d64")
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1
    assert "single_d64" in cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_rank_sequences_weak_and_strong():
    one = W.WORKLOADS["qwen_cache_r05"]
    assert one.n_seq == 1
    for world in (1, 2, 8):
        seen = [bench.rank_sequences(one, r, world) for r in range(world)]
        assert all(s == ([r], "weak") for r, s in enumerate(seen))
    many = W.WORKLOADS["longctx"]
    assert many.n_seq > 1
    for world in (1, 2, 4, 8):
        if many.n_seq % world:
            continue
        parts = [bench.rank_sequences(many, r, world) for r in range(world)]
        assert all(kind == "strong" for _, kind in parts)
        flat = sorted(x for seqs, _ in parts for x in seqs)
        assert flat == list(range(many.n_seq))  # every sequence exactly once
    with pytest.raises(SystemExit):
        bench.rank_sequences(many, 0, many.n_seq + 1 if many.n_seq > 1 else 3)


def test_recorded_traffic_guard(tmp_path, monkeypatch):
    h = bench.kernel_source_hash()
    rec = tmp_path / "traffic.md"
    rec.write_text(f"- workload: qwen_cache_r05\n- source_sha256: {h}\n"
                   "- dram_bytes_per_launch: 1234\n")
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(rec))
    assert bench.recorded_traffic("qwen_cache_r05") == 1234
    assert bench.recorded_traffic("qwen_cache_r03") is None  # another workload
    rec.write_text("- workload: qwen_cache_r05\n- source_sha256: " + "0" * 64 +
                   "\n- dram_bytes_per_launch: 1234\n")
    assert bench.recorded_traffic("qwen_cache_r05") is None  # sources changed since
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "missing.md"))
    assert bench.recorded_traffic("qwen_cache_r05") is None



def test_reference_arm_under_torchrun_prints_once():
    # two ranks: rank 0 alone times the oracle and prints; the other exits 0 without work
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
                        "--nproc-per-node", "2", "--master-addr", "127.0.0.1",
                        "--master-port", str(port), os.path.join(ROOT, "bench.py"),
                        "--impl", "reference", "--gpus", "2", "--workload", "single_d64",
                        "--steps", "1", "--warmup", "0", "--cpu-budget", "2"],
                       capture_output=True, text=True, timeout=900, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2
