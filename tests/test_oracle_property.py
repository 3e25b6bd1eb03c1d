"""Property-based pinning of the CPU oracle: on random small shapes (ragged N, GQA group sizes,
block sizes, k from 1 to more than the visible blocks, integer and normal index inputs) the
oracle's selection equals the dense numpy brute force and its attention equals dense attention
under that selection's mask."""
import numpy as np
import pytest

hypothesis = pytest.importorskip("hypothesis")
from hypothesis import given, settings  # noqa: E402
from hypothesis import strategies as st  # noqa: E402

import oracle  # noqa: E402
from block_sparse_long_idx_b200.synth import int_uniform_bf16, normal_bf16  # noqa: E402
from tests import ref_numpy as ref  # noqa: E402

shapes = st.tuples(
    st.integers(1, 160),            # N
    st.sampled_from([1, 2]),        # H_kv
    st.sampled_from([1, 2, 4]),     # G
    st.sampled_from([4, 8]),        # d_h
    st.sampled_from([4, 8]),        # d_idx
    st.sampled_from([4, 8, 16]),    # B_k
    st.integers(1, 6),              # k
    st.booleans(),                  # integer index inputs
    st.integers(0, 10_000),         # seed
)


@settings(max_examples=40, deadline=None, derandomize=True)
@given(shapes)
def test_oracle_matches_dense_brute_force(shape):
    N, H_kv, G, d_h, d_idx, B_k, k, integer, seed = shape
    H_q = H_kv * G
    if integer:
        qi = int_uniform_bf16((N, H_kv, d_idx), -3, 3, seed, "pqi")
        ki = int_uniform_bf16((N, H_kv, d_idx), -3, 3, seed, "pki")
    else:
        qi = normal_bf16((N, H_kv, d_idx), seed, "pqi")
        ki = normal_bf16((N, H_kv, d_idx), seed, "pki")
    inp = {"q_idx": qi, "k_idx": ki, "q": normal_bf16((N, H_q, d_h), seed, "pq"),
           "k": normal_bf16((N, H_kv, d_h), seed, "pk"), "v": normal_bf16((N, H_kv, d_h), seed, "pv")}
    rows = np.arange(N)
    sel, out, lse = oracle.prefill_rows(inp, rows, B_k, k)
    sel_r = np.ascontiguousarray(sel.transpose(1, 0, 2))
    assert np.array_equal(sel_r, ref.dense_selection(qi, ki, B_k, k))
    want, want_lse = ref.masked_attention(inp["q"], inp["k"], inp["v"], ref.selection_mask(sel_r, N, B_k))
    assert np.max(np.abs(out - want)) < 1e-12
    assert np.max(np.abs(lse - want_lse)) < 1e-12
