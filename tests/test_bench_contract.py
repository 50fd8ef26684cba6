"""The bench.py JSON line contract, checked on CPU through the reference
(oracle) arm on the tiny workload: every key the driver reads is present,
with the oracle's CPU baseline and an e2e object of zero transfer bytes."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = ["metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
        "scaling", "vs_baseline", "dtype", "data", "config"]


def _run(*extra):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0", *extra],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    return json.loads(lines[0])


def test_reference_arm_line_has_the_contract_keys():
    j = _run("--workload", "tiny")
    for k in KEYS:
        assert k in j, k
    assert j["impl"] == "reference" and j["value"] > 0 and j["higher_is_better"] is True
    assert j["scaling"] == "weak" and j["vs_baseline"] is None and j["data"] == "synthetic"
    cb = j["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == j["value"] and cb["sample"]
    assert j["e2e"] == {"value": j["value"], "unit": j["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    cfg = j["config"]
    assert cfg["workload"].startswith("tiny:") and cfg["fmt"] == "nvfp4" and cfg["nm"] == "2:4"
    assert "model" not in cfg


def test_reference_arm_follows_format_and_residual_options():
    j = _run("--workload", "tiny", "--fmt", "mxfp4", "--nm", "1:4", "--residual", "shared")
    assert j["config"]["fmt"] == "mxfp4" and j["config"]["nm"] == "1:4"
    assert j["config"]["residual_scale"] == "shared"


def test_reference_arm_runs_the_fused_mlp():
    j = _run("--workload", "tiny_mlp", "--fuse-mlp")
    assert j["config"]["mlp"].startswith("producer-fused") and j["value"] > 0
    assert "SwiGLU" in j["cpu_baseline"]["sample"]


def test_fused_mlp_needs_gate_up_and_down():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny", "--fuse-mlp", "--steps", "1", "--warmup", "0"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode != 0 and "gate_up and down" in out.stderr


def test_reference_arm_runs_the_fused_moe_layer():
    j = _run("--workload", "qwen3moe", "--fuse-mlp")
    assert j["config"]["mlp"].startswith("producer-fused") and j["value"] > 0
    assert "SwiGLU" in j["cpu_baseline"]["sample"]


def test_reference_arm_runs_the_pair_backbone():
    j = _run("--workload", "tiny", "--fmt", "mxfp4", "--nm", "4:8p")
    assert j["config"]["nm"] == "4:8p" and j["config"]["backbone"].startswith("pair-granular")
    assert "pair-granular" in j["cpu_baseline"]["sample"] and j["value"] > 0


def test_pair_backbone_needs_mxfp4():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny", "--nm", "4:8p", "--steps", "1", "--warmup", "0"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode != 0 and "MXFP4" in out.stderr
