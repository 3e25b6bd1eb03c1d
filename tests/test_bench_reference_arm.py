"""bench.py's reference arm (the oracle timed on host cores) on the tiny configuration: one JSON line
with the contract's keys, the prefill rate and the decode rate of the oracle."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_tiny():
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny_prefill_N2048",
           "--decode-workload", "decode_B64_L2K-16K", "--steps", "1", "--warmup", "0", "--cpu-seconds", "1"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["dtype"] == "f64" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["steps"] == 1 and d["warmup"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == "tiny_prefill_N2048 + decode_B64_L2K-16K"
    dec = d["decode"]
    assert dec["value"] > 0 and dec["unit"] == "tokens/s" and "4 sequences" in dec["sample"]
