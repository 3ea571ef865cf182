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
    assert d["metric"] == bench.metric_for(W.WORKLOADS["single_d64"])
    assert d["unit"] == "head-problems/s" and d["extrapolated"] is True
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


def test_gpus_flag_launches_the_ranks_itself():
    # without torchrun, --gpus 2 starts two processes with their own rank environment;
    # rank 0 alone prints the line, which reports both ranks
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--workload", "single_d64", "--steps", "1", "--warmup",
                        "0"], capture_output=True, text=True, timeout=900, cwd=ROOT,
                       env={k: v for k, v in os.environ.items() if k not in
                            ("RANK", "WORLD_SIZE", "LOCAL_RANK")})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2


def test_rank_env():
    base = {"PATH": "/bin", "RANK": "7"}
    envs = [bench.rank_env(base, 4, r, 29500) for r in range(4)]
    assert [e["RANK"] for e in envs] == ["0", "1", "2", "3"]
    assert [e["LOCAL_RANK"] for e in envs] == ["0", "1", "2", "3"]
    assert all(e["WORLD_SIZE"] == "4" and e["MASTER_ADDR"] == "127.0.0.1" and
               e["MASTER_PORT"] == "29500" and e["PATH"] == "/bin" for e in envs)
    assert base["RANK"] == "7"  # the caller's environment is left alone


def test_spawn_reports_a_failing_rank(tmp_path, monkeypatch):
    script = tmp_path / "fail_rank1.py"
    script.write_text("import os, sys\nsys.exit(3 if os.environ['RANK'] == '1' else 0)\n")
    monkeypatch.setattr(bench, "__file__", str(script))
    assert bench.spawn_ranks(2, [], timeout_s=120) == 3


def test_metric_labels():
    assert bench.metric_for(W.WORKLOADS["qwen_cache_r05"]) == bench.METRIC
    assert bench.metric_for(W.WORKLOADS["qwen_cache_r03"]).endswith("N=2048,r=0.3")
    assert bench.metric_for(W.WORKLOADS["qwen_cache_r07"]).endswith("N=2048,r=0.7")
    assert bench.metric_for(W.WORKLOADS["longctx"]).endswith("N=8192,r=0.3")
    assert "adaptive" in bench.metric_for(W.WORKLOADS["qwen_cache_adaptive"])
