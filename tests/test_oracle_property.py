"""Property-based pinning of the CPU oracle: on random small shapes (ragged N, GQA group sizes,
block sizes, k from 1 to more than the visible blocks, integer and normal index inputs) the
oracle's selection equals the dense numpy brute force and its attention equals dense attention
under that selection's mask; its backward (main-branch gradients, KL alignment and its gradients)
equals autograd of the masked dense definitions."""
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


@settings(max_examples=25, deadline=None, derandomize=True)
@given(shapes)
def test_oracle_backward_matches_autograd(shape):
    """The oracle's hand-derived gradients (main branch and KL alignment) equal autograd of the
    masked dense definitions on random small shapes."""
    from tests import ref_autograd

    N, H_kv, G, d_h, d_idx, B_k, k, integer, seed = shape
    N = min(N, 96)
    H_q = H_kv * G
    gen = int_uniform_bf16 if integer else None
    qi = gen((N, H_kv, d_idx), -3, 3, seed, "bqi") if gen else normal_bf16((N, H_kv, d_idx), seed, "bqi")
    ki = gen((N, H_kv, d_idx), -3, 3, seed, "bki") if gen else normal_bf16((N, H_kv, d_idx), seed, "bki")
    q, kk, v = (normal_bf16((N, H, d_h), seed, n) for H, n in ((H_q, "bq"), (H_kv, "bk"), (H_kv, "bv")))
    dout = normal_bf16((N, H_q, d_h), seed, "bdo")
    rows = np.arange(N)
    sel = oracle.select_rows(qi, ki, rows, B_k, k)
    allowed = ref.selection_mask(np.ascontiguousarray(sel.transpose(1, 0, 2)), N, B_k)
    nb = (N + B_k - 1) // B_k
    pairs = [(r, b) for r in range(H_kv) for b in range(nb)]
    tok = lambda g: g.reshape(H_kv, nb * B_k, -1)[:, :N].transpose(1, 0, 2)  # noqa: E731

    dq = oracle.backward_dq_rows(q, dout, kk, v, rows, sel, B_k)
    dk, dv = oracle.backward_dkv_blocks(q, dout, kk, v, sel, pairs, B_k)
    wq, wk, wv = ref_autograd.attention_grads(q, kk, v, dout, allowed)
    for got, want in ((dq, wq), (tok(dk), wk), (tok(dv), wv)):
        assert np.max(np.abs(got - want)) < 1e-10

    w = 1.0 / (N * H_kv)
    kl, dqi = oracle.kl_rows(q, qi, kk, ki, rows, sel, B_k, w)
    dki = oracle.kl_dk_idx_blocks(q, qi, kk, ki, sel, pairs, B_k, w)
    wkl, wqi, wki = ref_autograd.kl_loss_grads(q, kk, qi, ki, allowed, w)
    assert np.max(np.abs(kl - wkl)) < 1e-9
    assert np.max(np.abs(dqi - wqi)) < 1e-12 and np.max(np.abs(tok(dki) - wki)) < 1e-12
