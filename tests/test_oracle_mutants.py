"""Plausible mistakes planted in a copy of the oracle must each fail at least one pin.

The copy is compiled into a temporary directory; the committed oracle is never modified.
"""
import os
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_RUNNER = """
import sys
sys.path.insert(0, {root!r})
import oracle
from tests import pins
o = oracle.Oracle({so!r})
failed = []
for check in pins.ALL_CHECKS:
    try:
        check(o)
    except (AssertionError, ValueError, IndexError):
        failed.append(check.__name__)
print("FAILED:" + ",".join(failed))
"""

# (name, text in msa_oracle.c, replacement)
MUTANTS = [
    ("tie_break_to_higher_block", "return (x->block > y->block) - (x->block < y->block);",
     "return (x->block < y->block) - (x->block > y->block);"),
    ("local_block_not_forced", "sel[n++] = (int32_t)local;", "if (take < k) sel[n++] = (int32_t)(local > 0 ? local - 1 : 0);"),
    ("scale_1_over_d", "const double scale = 1.0 / sqrt((double)d_h);", "const double scale = 1.0 / (double)d_h;"),
    ("causal_strict", "j < ((int64_t)b + 1) * B_k && j <= i; ++j) {\n            const uint16_t* kr",
     "j < ((int64_t)b + 1) * B_k && j < i; ++j) {\n            const uint16_t* kr"),
    ("pool_sum_not_max", "if (s > best) best = s; /* block max pooling */",
     "best = (best == -INFINITY ? 0.0 : best) + s;"),
    ("k_not_counting_local", "(int64_t)(k - 1);\n    for (int64_t t = 0; t < take",
     "(int64_t)(k);\n    for (int64_t t = 0; t < take"),
    ("wrong_gqa_group", "const int r = h / G;", "const int r = h % H_kv;"),
    ("lse_missing_max", "*lse = m + log(z);", "*lse = log(z);"),
    ("kv2q_slot_off_by_one", "ent[fill[b]++] = (int32_t)(i * k + s);", "ent[fill[b]++] = (int32_t)(i * k + s + 1);"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    src = open(oracle.SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    src = src.replace(old, new)
    if name == "k_not_counting_local":  # k non-local blocks, the local one only if room is left
        src = src.replace("sel[n++] = (int32_t)local;", "if (n < k) sel[n++] = (int32_t)local;")
    path = tmp_path / "mutant.c"
    path.write_text(src)
    so = oracle.compile_oracle(str(path), str(tmp_path / "mutant.so"), force=True)
    # run in a child process: a mutant may also crash, which counts as caught
    proc = subprocess.run([sys.executable, "-c", _RUNNER.format(root=ROOT, so=so)], capture_output=True, text=True,
                          timeout=600)
    lines = [l for l in proc.stdout.splitlines() if l.startswith("FAILED:")]
    caught = proc.returncode != 0 or (lines and lines[-1] != "FAILED:")
    assert caught, f"mutant {name} passed every pin"
