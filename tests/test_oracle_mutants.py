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
    ("scale_1_over_d", "const double scale = 1.0 / sqrt((double)d_h);\n    double q[512];",
     "const double scale = 1.0 / (double)d_h;\n    double q[512];"),
    ("bwd_logits_scale_1_over_d",
     "const double scale = 1.0 / sqrt((double)d_h);\n    int64_t n = 0;\n    double m = -INFINITY;\n"
     "    for (int s = 0; s < k; ++s) {\n        int32_t b",
     "const double scale = 1.0 / (double)d_h;\n    int64_t n = 0;\n    double m = -INFINITY;\n"
     "    for (int s = 0; s < k; ++s) {\n        int32_t b"),
    ("causal_strict", "j <= i; ++j) {\n            const uint16_t* kr = kseq + ((size_t)j * H_kv + r) * d_h;\n            double dot = 0.0;\n            for (int d = 0; d < d_h; ++d) dot += q[d] * bf16_to_double(kr[d]);\n            logits[n]",
     "j < i; ++j) {\n            const uint16_t* kr = kseq + ((size_t)j * H_kv + r) * d_h;\n            double dot = 0.0;\n            for (int d = 0; d < d_h; ++d) dot += q[d] * bf16_to_double(kr[d]);\n            logits[n]"),
    ("bwd_causal_strict", "j <= i; ++j) {\n            const uint16_t* kr = kseq + ((size_t)j * H_kv + r) * d_h;\n            double dot = 0.0;\n            for (int d = 0; d < d_h; ++d) dot += q[d] * bf16_to_double(kr[d]);\n            p[n]",
     "j < i; ++j) {\n            const uint16_t* kr = kseq + ((size_t)j * H_kv + r) * d_h;\n            double dot = 0.0;\n            for (int d = 0; d < d_h; ++d) dot += q[d] * bf16_to_double(kr[d]);\n            p[n]"),
    ("pool_sum_not_max", "if (s > best) best = s; /* block max pooling */",
     "best = (best == -INFINITY ? 0.0 : best) + s;"),
    ("k_not_counting_local", "(int64_t)(k - 1);\n    for (int64_t t = 0; t < take",
     "(int64_t)(k);\n    for (int64_t t = 0; t < take"),
    ("wrong_gqa_group", "const int r = h / G;\n                    attend_one(",
     "const int r = h % H_kv;\n                    attend_one("),
    ("bwd_wrong_gqa_group", "const int r = h / G;\n                    double qd[512], dod[512];",
     "const int r = h % H_kv;\n                    double qd[512], dod[512];"),
    ("lse_missing_max", "*lse = m + log(z);\n}\n\n/*\n *   q    :", "*lse = log(z);\n}\n\n/*\n *   q    :"),
    ("e4m3_lse_missing_max", "*lse = m + log(z);\n}\n\n/*\n * (3) on E4M3", "*lse = log(z);\n}\n\n/*\n * (3) on E4M3"),
    ("kv2q_slot_off_by_one", "ent[fill[b]++] = (int32_t)(i * k + s);", "ent[fill[b]++] = (int32_t)(i * k + s + 1);"),
    ("bwd_softmax_jacobian_without_D", "ds[t] = p[t] * (dp - D);", "ds[t] = p[t] * dp;"),
    ("bwd_dk_from_dout", "gk[jj * d_h + d] += scale * ds[u] * qd[d];", "gk[jj * d_h + d] += scale * ds[u] * dod[d];"),
    ("bwd_dv_unweighted", "gv[jj * d_h + d] += p[u] * dod[d];", "gv[jj * d_h + d] += dod[d];"),
    ("bwd_dq_unscaled", "for (int d = 0; d < d_h; ++d) g[d] += scale * ds[u] * bf16_to_double(kr[d]);",
     "for (int d = 0; d < d_h; ++d) g[d] += ds[u] * bf16_to_double(kr[d]);"),
    ("kl_teacher_summed_not_averaged", "P[t] = (h == r * G ? 0.0 : P[t]) + p[t] / G;",
     "P[t] = (h == r * G ? 0.0 : P[t]) + p[t];"),
    ("kl_gradient_sign", "const double gs = w * (exp(lq[u]) - P[u]);\n                        const uint16_t* kr",
     "const double gs = w * (P[u] - exp(lq[u]));\n                        const uint16_t* kr"),
    ("kl_student_scaled", "lq[t] = s;\n", "lq[t] = s / sqrt((double)d_idx);\n"),
    ("e4m3_ties_to_odd", "(dc == db && (c & 1) == 0)", "(dc == db && (c & 1) == 1)"),
    ("e4m3_exponent_bias_8", "ldexp((double)(8 + m), e - 10)", "ldexp((double)(8 + m), e - 11)"),
    ("e4m3_scale_over_240", "amax > 0.0 ? amax / 448.0 : 1.0", "amax > 0.0 ? amax / 240.0 : 1.0"),
    ("e4m3_value_scale_dropped", "kd[x * d_h + d] = msa_oracle_e4m3_decode(kc[x * d_h + d]) * ks[x];",
     "kd[x * d_h + d] = msa_oracle_e4m3_decode(kc[x * d_h + d]);"),
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
