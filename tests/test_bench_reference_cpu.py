"""The reference arm of bench.py (the CPU oracle, timed on the host cores) runs
without a GPU and prints one JSON line of the agreed shape."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--cpu-seconds", "1"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT,
                       env={**os.environ, "CUDA_VISIBLE_DEVICES": ""})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [line for line in r.stdout.splitlines() if line.strip()]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["steps"] == 1 and d["warmup"] == 3
    assert d["config"]["workload"] == "rfq_linear_dit_ffn_M32768_K5120_N13824"
    # ms_per_step is the measured host time of a step's sample, not an extrapolation
    assert 0 < d["ms_per_step"] < 60e3 and d["extrapolated_ms_per_full_step"] > d["ms_per_step"]
    cb = d["cpu_baseline"]
    assert cb["threads"]["quantize_c_openmp"] >= 1
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_print_nothing():
    """Under torchrun only rank 0 runs the reference arm; the others exit 0 without work."""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--cpu-seconds", "1"],
                       capture_output=True, text=True, timeout=120, cwd=ROOT,
                       env={**os.environ, "CUDA_VISIBLE_DEVICES": "", "RANK": "1", "LOCAL_RANK": "1",
                            "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
