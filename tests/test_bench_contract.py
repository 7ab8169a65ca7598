"""bench.py's JSON line, checked on the CPU through its reference arm (the oracle on the host
cores; the GPU arm needs a device): one JSON line on stdout with the contract's keys, the
oracle described as the baseline, and an e2e entry with no host-device traffic."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    return json.loads(lines[0])


def test_reference_arm_line():
    r = _run("--impl", "reference", "--workload", "small_fp8", "--steps", "2", "--warmup", "3")
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "e2e",
                "cpu_baseline"):
        assert key in r, key
    assert r["impl"] == "reference"
    assert (r["n_gpus"], r["steps"], r["warmup"]) == (1, 2, 3)
    assert r["higher_is_better"] is True and r["value"] > 0 and r["ms_per_step"] > 0
    assert "workload" in r["config"]
    cb = r["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == r["value"] and cb["sample"]
    e2e = r["e2e"]
    assert (e2e["value"], e2e["unit"]) == (r["value"], r["unit"])
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_warmup_below_three_is_refused():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--warmup", "2"], capture_output=True, text=True, timeout=120, cwd=ROOT)
    assert out.returncode != 0 and "warmup" in out.stderr
