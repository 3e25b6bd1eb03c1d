"""The roofline's analytic FLOP model against the numbers the pages print (tests/golden/flop_ratio.txt)."""
import os

from block_sparse_long_idx_b200 import roofline

HERE = os.path.dirname(os.path.abspath(__file__))


def _golden():
    vals = {}
    for line in open(os.path.join(HERE, "golden", "flop_ratio.txt")):
        line = line.strip()
        if line and not line.startswith("#"):
            key, val = line.split()
            vals[key] = float(val)
    return vals


def test_flop_reduction_at_1m_matches_page():
    g = _golden()
    N, H_q, H_kv, d_h, d_idx, k, B_k = (int(g[x]) for x in ("N", "H_q", "H_kv", "d_h", "d_idx", "k", "B_k"))
    ratio = roofline.gqa_flops(N, H_q, d_h) / roofline.msa_flops(N, H_q, H_kv, d_h, d_idx, k, B_k)
    assert round(ratio, 1) == g["flop_reduction"]


def test_arithmetic_intensities_match_page():
    """KV-outer: a 128-row tile against one K/V block, 4*128*B_k*d FLOP over 3 bf16 tiles of 128 x d;
    Q-outer: one position's G rows against one block, 4*G*B_k*d FLOP over K, V and G query rows."""
    g = _golden()
    B_k, d, G = 128, 128, 16
    kv_outer = 4 * 128 * B_k * d / (2 * 3 * 128 * d)
    q_outer = 4 * G * B_k * d / (2 * (2 * B_k * d + G * d))
    assert round(kv_outer) == g["kv_outer_intensity"]
    # the page quotes the leading-order value G; the exact ratio is G / (1 + G / (2 * B_k))
    assert abs(q_outer - g["q_outer_intensity"]) / g["q_outer_intensity"] < 0.1


def test_main_branch_budget_is_linear_in_n():
    a = roofline.main_branch_flops(2 ** 17, 64, 128, 16, 128)
    b = roofline.main_branch_flops(2 ** 20, 64, 128, 16, 128)
    assert b / a == 8.0


def test_backward_flops_are_five_products():
    """Backward with the selections fixed: per (row, head, selected block) the recomputed S and the
    dP, dV, dK, dQ products, five B_k x d_h contractions of 2 FLOP per multiply-add against the
    forward's two."""
    N, H_q, d_h, k, B_k = 2 ** 17, 64, 128, 16, 128
    per_unit = 5 * 2 * B_k * d_h
    assert roofline.main_branch_backward_flops(N, H_q, d_h, k, B_k) == per_unit * N * H_q * k
    assert roofline.main_branch_backward_flops(N, H_q, d_h, k, B_k) == 2.5 * roofline.main_branch_flops(N, H_q, d_h,
                                                                                                          k, B_k)
