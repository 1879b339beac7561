"""The benchmark's JSON contract, checked on the CPU: the reference arm (the
fp64 oracle on the host cores) runs end to end on a small workload and prints
one line with every key the contract names; both arms describe a workload with
the same config builder."""
import json
import os
import subprocess
import sys

import bench
from rope_block_sparse_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

BASE_KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
             "vs_baseline", "dtype", "data", "config"}


def test_reference_arm_prints_one_contract_line():
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "3",
           "--ref-rows", "8"]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, res.stdout
    d = json.loads(lines[0])
    assert BASE_KEYS <= set(d) and d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["steps"] == 2 and d["warmup"] == 3 and d["n_gpus"] == 1 and d["value"] > 0
    assert d["vs_baseline"] is None and d["data"] == "synthetic"
    assert d["config"] == bench.config_of(synth.WORKLOADS["tiny"], 1, 1)
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and "8 sampled" in cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_refuses_short_warmup():
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "2"]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=120)
    assert res.returncode != 0 and "at least 3" in res.stderr


def test_config_names_the_workload_not_a_model():
    w = synth.WORKLOADS[bench.WORKLOAD]
    c = bench.config_of(w, 8, 245)
    assert "model" not in c
    assert c["workload"].startswith("video5s_sparse: B=1, 56 heads x 96, grid 31x48x84 = 124,992 tokens")
    assert "k=245/977" in c["workload"] and c["parallelism"].startswith("dp8")
    assert c["tokens"] == 124992 and c["heads"] == 56 and c["head_dim"] == 96 and c["sparsity"] == bench.SPARSITY
    assert c["l2"].startswith("inputs larger than L2")


def _free_port() -> int:
    import socket

    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_reference_arm_under_torchrun_prints_once():
    """Two ranks launched the way the multi-GPU bench is: rank 0 alone runs the
    oracle and prints; the other rank exits 0 without work."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--impl", "reference",
           "--gpus", "2", "--workload", "tiny", "--steps", "1", "--warmup", "3", "--ref-rows", "8"]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1, res.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["config"]["parallelism"].startswith("dp2")


def test_end_to_end_pass_runs_the_timed_step_count_unless_told_otherwise():
    assert bench.parse_args(["--steps", "20", "--warmup", "3"]).e2e_steps == 20
    assert bench.parse_args([]).e2e_steps == bench.parse_args([]).steps
    assert bench.parse_args(["--steps", "7", "--e2e-steps", "0"]).e2e_steps == 0
