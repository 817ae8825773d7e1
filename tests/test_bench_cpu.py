"""bench.py's reference arm (the fp64 oracle on the host's cores) runs without a
GPU and prints the contract's JSON line."""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--config", "2", "--steps", "1", "--warmup", "3",
                        "--reference-budget-s", "1"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "TFLOP/s"
    assert d["higher_is_better"] is True and d["n_gpus"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"].startswith("short_history")
    c = d["config"]
    for key in ("B", "total_tokens", "max_seqlen", "num_pos", "num_time_buckets", "seed", "H",
                "d", "l2"):
        assert key in c, key
    assert c["seed"] == 1002 and c["num_pos"] == 200 and c["num_time_buckets"] == 128
    # ms_per_step is a measured wall time of one sampled step; the whole-batch
    # time is extrapolated under its own key
    assert 0 < d["ms_per_step"] < 600e3
    assert d["ms_per_full_batch_extrapolated"] > 0


def test_reference_arm_layer_workload():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--config", "5", "--steps", "1", "--warmup", "3",
                        "--reference-budget-s", "1"],
                       capture_output=True, text=True, timeout=900, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads([ln for ln in r.stdout.splitlines() if ln.strip()][0])
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["config"]["workload"].startswith("layer_") and d["config"]["D"] == 512
