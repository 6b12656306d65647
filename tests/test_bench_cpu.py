"""bench.py's JSON contract on the host: the reference arm (the oracle timed
on the host cores) prints exactly one line with every key the driver reads,
and the measured arm refuses to run without a GPU instead of falling back to
the CPU."""

import json
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _bench(*args, timeout=600):
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                          capture_output=True, text=True, timeout=timeout)


def test_reference_arm_prints_one_complete_line():
    import bench
    p = _bench("--impl", "reference", "--steps", "3", "--warmup", "3")
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["value"] > 0 and d["steps"] == 3 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["higher_is_better"] is True and d["vs_baseline"] is None
    assert d["data"] == "synthetic" and "workload" in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the behaviour without a GPU")
def test_measured_arm_refuses_to_run_without_a_gpu():
    p = _bench("--steps", "3", "--warmup", "3")
    assert p.returncode != 0
    assert not [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert "needs a CUDA GPU" in p.stderr


def test_traffic_hash_follows_code_not_comments(tmp_path):
    import bench
    a = tmp_path / "a.cu"
    a.write_text("// header\nint f(int x) {\n  return x + 1;  // one\n}\n")
    h = bench.source_code_hash(str(a))
    a.write_text("/* another\n   header */\n\nint f(int x) {\n    return x + 1;\n}\n")
    assert bench.source_code_hash(str(a)) == h         # comments and layout only
    a.write_text("// header\nint f(int x) {\n  return x + 2;  // one\n}\n")
    assert bench.source_code_hash(str(a)) != h         # a code change


def test_reference_arm_under_torchrun_prints_once():
    # the driver launches every N > 1 arm through torch.distributed.run; on
    # the host the ranks join over gloo, rank 0 alone runs the oracle and
    # prints, the others leave without work, and every rank exits 0
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    p = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
                        "--nproc-per-node", "2", "--master-addr", "127.0.0.1", "--master-port",
                        str(port), os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "2", "--warmup", "3"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
