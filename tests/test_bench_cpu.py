"""bench.py's reference arm (the CPU oracle on the bench's metric) keeps the
JSON contract, on the CPU: one line with the metric, unit, step counts, the
measured time of the samples it ran as the step time, the extrapolated rate
as the value (marked as such, with the full step time it implies), the
oracle's cpu_baseline and an e2e object with no host copies."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--shape", "tiny", "--batch", "2",
                        "--seq", "64", "--steps", "2", "--warmup", "1"], cwd=ROOT, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tok/s" and d["value"] > 0
    assert (d["n_gpus"], d["steps"], d["warmup"]) == (1, 2, 1)
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["vs_baseline"] is None
    assert d["dtype"] == "f64" and d["data"] == "synthetic" and "workload" in d["config"]
    assert d["value_basis"] == "extrapolated" and d["samples_run"] == 3
    assert abs(d["extrapolated_ms_per_full_step"] - 2 * 64 / d["value"] * 1e3) <= 1e-6 * d["extrapolated_ms_per_full_step"]
    assert 0 < d["ms_per_step"] < 600e3
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
