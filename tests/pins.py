"""Pin checks for the CPU oracle.

Each check takes an ``oracle.Oracle`` instance and raises AssertionError on a mismatch. They
pin the oracle to things other than itself: a dense brute force on tiny inputs, closed forms,
textbook dense attention when the budget covers the whole context, invariants of the selected
sets, and the split-then-merge identity. ``test_oracle_pins`` runs them on the real oracle and
``test_oracle_mutants`` shows that each plausible mistake planted in a copy of the oracle fails
at least one of them.
"""
from __future__ import annotations

import math

import numpy as np

from block_sparse_long_idx_b200.synth import bf16_bits_to_f64, f32_to_bf16_bits, int_uniform_bf16, normal_bf16
from tests import ref_autograd
from tests import ref_numpy as ref

# (N, H_q, H_kv, d_h, d_idx, B_k, k) -- small shapes spanning several blocks, ragged tails, k larger
# than the number of visible blocks, G = 1 and G > 1.
SEL_SHAPES = [
    (1, 2, 1, 8, 4, 4, 2),
    (37, 4, 2, 8, 8, 4, 3),
    (64, 2, 2, 8, 16, 8, 4),
    (130, 4, 1, 16, 8, 16, 5),
    (300, 8, 2, 8, 32, 16, 8),
    (517, 2, 1, 8, 8, 32, 4),
]


def _idx_inputs(N, H_kv, d_idx, seed, integer=True):
    shp = (N, H_kv, d_idx)
    if integer:
        return int_uniform_bf16(shp, -3, 3, seed, "pq"), int_uniform_bf16(shp, -3, 3, seed, "pk")
    return normal_bf16(shp, seed, "pq"), normal_bf16(shp, seed, "pk")


def check_selection_bruteforce(o):
    """Selection equals the dense brute force exactly (integer and non-integer index inputs)."""
    for t, (N, _, H_kv, _, d_idx, B_k, k) in enumerate(SEL_SHAPES):
        for integer in (True, False):
            qi, ki = _idx_inputs(N, H_kv, d_idx, 100 + t, integer)
            got = o.select_all(qi, ki, B_k, k)
            want = ref.dense_selection(qi, ki, B_k, k)
            assert np.array_equal(got, want), f"selection mismatch at shape {t} integer={integer}"


def check_selection_ties_closed_form(o):
    """q_idx == 0 makes every score 0: the set is the lowest k-1 visible blocks plus the local block."""
    N, H_kv, d_idx, B_k, k = 200, 2, 8, 8, 5
    qi = np.zeros((N, H_kv, d_idx), dtype=np.uint16)  # +0.0 in bf16
    ki = int_uniform_bf16((N, H_kv, d_idx), -3, 3, 7, "tk")
    got = o.select_all(qi, ki, B_k, k)
    for i in range(N):
        loc = i // B_k
        want = sorted(set(range(min(k - 1, loc))) | {loc})
        want = want + [-1] * (k - len(want))
        for r in range(H_kv):
            assert list(got[r, i]) == want, (i, r, list(got[r, i]), want)


def check_selection_planted_winners(o):
    """Blocks with k_idx = +3 (winners) beat blocks with k_idx = 0 when q_idx = +1; ties go lower."""
    N, H_kv, d_idx, B_k, k = 256, 1, 4, 8, 4
    nb = N // B_k
    winners = {3, 5, 6, 11, 17, 18, 25, 30}
    qi = f32_to_bf16_bits(np.ones((N, H_kv, d_idx), dtype=np.float32))
    kf = np.zeros((N, H_kv, d_idx), dtype=np.float32)
    for b in winners:
        kf[b * B_k:(b + 1) * B_k] = 3.0
    ki = f32_to_bf16_bits(kf)
    got = o.select_all(qi, ki, B_k, k)[0]
    for i in range(N):
        loc = i // B_k
        vis_w = [b for b in sorted(winners) if b < loc]
        vis_o = [b for b in range(loc) if b not in winners]
        pick = (vis_w + vis_o)[: k - 1]
        want = sorted(pick + [loc])
        want = want + [-1] * (k - len(want))
        assert list(got[i]) == want, (i, list(got[i]), want)
    assert nb == 32


def check_selection_invariants(o):
    """Local block kept, |set| = min(k, local+1), ascending, distinct, visible, -1 padding last."""
    N, H_kv, d_idx, B_k, k = 700, 2, 16, 16, 6
    qi, ki = _idx_inputs(N, H_kv, d_idx, 11)
    sel = o.select_all(qi, ki, B_k, k)
    for r in range(H_kv):
        for i in range(N):
            s = list(sel[r, i])
            loc = i // B_k
            n = min(k, loc + 1)
            assert all(x >= 0 for x in s[:n]) and all(x == -1 for x in s[n:]), (r, i, s)
            v = s[:n]
            assert v == sorted(set(v)) and loc in v and max(v) == loc and min(v) >= 0, (r, i, s)


def _attn_inputs(N, H_q, H_kv, d_h, d_idx, seed):
    return {
        "q": normal_bf16((N, H_q, d_h), seed, "aq"),
        "k": normal_bf16((N, H_kv, d_h), seed, "ak"),
        "v": normal_bf16((N, H_kv, d_h), seed, "av"),
        "q_idx": int_uniform_bf16((N, H_kv, d_idx), -3, 3, seed, "aqi"),
        "k_idx": int_uniform_bf16((N, H_kv, d_idx), -3, 3, seed, "aki"),
    }


def check_attention_dense_invariant(o):
    """When k*B_k >= N every visible block is selected, so MSA equals dense causal GQA attention."""
    for (N, H_q, H_kv, d_h, B_k, k) in [(64, 4, 2, 16, 16, 4), (100, 4, 1, 8, 8, 13), (96, 8, 2, 32, 32, 3)]:
        inp = _attn_inputs(N, H_q, H_kv, d_h, 8, N)
        rows = np.arange(N)
        sel, out, lse = o.prefill_rows(inp, rows, B_k, k)
        want, want_lse = ref.dense_causal_gqa(inp["q"], inp["k"], inp["v"])
        assert np.max(np.abs(out - want)) < 1e-12, np.max(np.abs(out - want))
        assert np.max(np.abs(lse - want_lse)) < 1e-12


def check_attention_masked_bruteforce(o):
    """With k*B_k < N, attention equals dense attention under the selection mask (brute force)."""
    N, H_q, H_kv, d_h, d_idx, B_k, k = 160, 4, 2, 16, 8, 16, 3
    inp = _attn_inputs(N, H_q, H_kv, d_h, d_idx, 5)
    rows = np.arange(N)
    sel, out, lse = o.prefill_rows(inp, rows, B_k, k)
    sel_r = np.ascontiguousarray(sel.transpose(1, 0, 2))
    assert np.array_equal(sel_r, ref.dense_selection(inp["q_idx"], inp["k_idx"], B_k, k))
    want, want_lse = ref.masked_attention(inp["q"], inp["k"], inp["v"], ref.selection_mask(sel_r, N, B_k))
    assert np.max(np.abs(out - want)) < 1e-12
    assert np.max(np.abs(lse - want_lse)) < 1e-12


def check_attention_zero_keys(o):
    """k == 0: all logits equal, so out is the plain mean of v over the attended tokens, lse = log|T|."""
    N, H_q, H_kv, d_h, d_idx, B_k, k = 90, 4, 2, 8, 8, 8, 3
    inp = _attn_inputs(N, H_q, H_kv, d_h, d_idx, 9)
    inp["k"] = np.zeros_like(inp["k"])
    rows = np.arange(N)
    sel, out, lse = o.prefill_rows(inp, rows, B_k, k)
    V = bf16_bits_to_f64(inp["v"])
    G = H_q // H_kv
    for t, i in enumerate(rows):
        for h in range(H_q):
            r = h // G
            toks = [j for b in sel[t, r] if b >= 0 for j in range(b * B_k, min((b + 1) * B_k, i + 1))]
            assert np.max(np.abs(out[t, h] - V[toks, r].mean(axis=0))) < 1e-12
            assert abs(lse[t, h] - math.log(len(toks))) < 1e-12


def check_attention_k1_block_local(o):
    """k = 1 keeps only the local block: causal attention inside each query's own block."""
    N, H_q, H_kv, d_h, d_idx, B_k = 70, 2, 1, 8, 8, 16
    inp = _attn_inputs(N, H_q, H_kv, d_h, d_idx, 13)
    rows = np.arange(N)
    sel, out, lse = o.prefill_rows(inp, rows, B_k, 1)
    blk = np.arange(N) // B_k
    allowed = (blk[:, None] == blk[None, :]) & np.tril(np.ones((N, N), dtype=bool))
    want, want_lse = ref.masked_attention(inp["q"], inp["k"], inp["v"], allowed[None])
    assert np.max(np.abs(out - want)) < 1e-12
    assert np.max(np.abs(lse - want_lse)) < 1e-12


def check_attention_hand_example(o):
    """Three tokens, d_h = 4 (scale 1/2), q = (2,0,0,0), k_j = (j,0,0,0): logits 0, 1, 2 at row 2.

    With v_j = (1, j, j^2, 0) the exact answer is (1, (e+2e^2)/Z, (e+4e^2)/Z, 0), Z = 1+e+e^2,
    lse = log Z (B_k = 2, k = 2: row 2 keeps block 0 and its local block 1)."""
    f = lambda a: f32_to_bf16_bits(np.asarray(a, dtype=np.float32))
    inp = {
        "q": f([[[2, 0, 0, 0]]] * 3),
        "k": f([[[0, 0, 0, 0]], [[1, 0, 0, 0]], [[2, 0, 0, 0]]]),
        "v": f([[[1, 0, 0, 0]], [[1, 1, 1, 0]], [[1, 2, 4, 0]]]),
        "q_idx": f(np.zeros((3, 1, 1))),
        "k_idx": f(np.zeros((3, 1, 1))),
    }
    sel, out, lse = o.prefill_rows(inp, np.array([0, 1, 2]), 2, 2)
    e = math.e
    Z = 1 + e + e * e
    assert list(sel[2, 0]) == [0, 1]
    want = np.array([1.0, (e + 2 * e * e) / Z, (e + 4 * e * e) / Z, 0.0])
    assert np.max(np.abs(out[2, 0] - want)) < 1e-14, out[2, 0]
    assert abs(lse[2, 0] - math.log(Z)) < 1e-14
    # row 1 attends tokens 0 and 1 (logits 0 and 1); row 0 only token 0
    Z1 = 1 + e
    assert np.max(np.abs(out[1, 0] - np.array([1.0, e / Z1, e / Z1, 0.0]))) < 1e-14
    assert np.max(np.abs(out[0, 0] - np.array([1.0, 0.0, 0.0, 0.0]))) < 1e-14
    assert abs(lse[0, 0]) < 1e-14


def check_combine_identity(o):
    """Per-block softmax partials merged through their log-sum-exp equal the one-pass result."""
    N, H_q, H_kv, d_h, d_idx, B_k, k = 200, 4, 2, 16, 8, 16, 4
    inp = _attn_inputs(N, H_q, H_kv, d_h, d_idx, 21)
    rows = np.array([0, 15, 16, 77, 130, 199])
    sel, out, lse = o.prefill_rows(inp, rows, B_k, k)
    Q, K, V = (bf16_bits_to_f64(inp[x]) for x in ("q", "k", "v"))
    G = H_q // H_kv
    for t, i in enumerate(rows):
        for h in range(H_q):
            r = h // G
            parts = []
            for b in sel[t, r]:
                if b < 0:
                    continue
                js = np.arange(b * B_k, min((b + 1) * B_k, i + 1))
                s = K[js, r] @ Q[i, h] / math.sqrt(d_h)
                m = s.max()
                w = np.exp(s - m)
                parts.append((m + math.log(w.sum()), (w / w.sum()) @ V[js, r]))
            L = np.logaddexp.reduce([p[0] for p in parts])
            merged = sum(math.exp(p[0] - L) * p[1] for p in parts)
            assert abs(L - lse[t, h]) < 1e-12
            assert np.max(np.abs(merged - out[t, h])) < 1e-12


def check_kv2q_bruteforce(o):
    """The inversion lists equal a per-block brute-force scan, for oracle selections."""
    N, H_kv, d_idx, B_k, k = 333, 2, 8, 16, 5
    qi, ki = _idx_inputs(N, H_kv, d_idx, 31)
    sel = o.select_all(qi, ki, B_k, k)
    off, ent = o.kv2q(sel, B_k)
    want = ref.brute_kv2q(sel, B_k)
    nb = (N + B_k - 1) // B_k
    for r in range(H_kv):
        for b in range(nb):
            assert np.array_equal(ent[r][off[r, b]:off[r, b + 1]], want[r][b]), (r, b)
        assert off[r, -1] == sum(min(k, i // B_k + 1) for i in range(N))


def check_decode_matches_prefill_row(o):
    """Decode of a sequence of length L equals prefill row L-1 of the same data."""
    B, L_max, H_q, H_kv, d_h, d_idx, B_k, k = 3, 150, 4, 2, 8, 8, 16, 3
    lens = np.array([1, 77, 150], dtype=np.int32)
    kc = normal_bf16((B, L_max, H_kv, d_h), 3, "dk")
    vc = normal_bf16((B, L_max, H_kv, d_h), 3, "dv")
    kic = int_uniform_bf16((B, L_max, H_kv, d_idx), -3, 3, 3, "dki")
    q = normal_bf16((B, H_q, d_h), 3, "dq")
    qi = int_uniform_bf16((B, H_kv, d_idx), -3, 3, 3, "dqi")
    dec = {"q": q, "q_idx": qi, "k_cache": kc, "v_cache": vc, "k_idx_cache": kic, "lens": lens}
    sel, out, lse = o.decode(dec, B_k, k)
    for beta in range(B):
        L = int(lens[beta])
        inp = {"k": kc[beta, :L], "v": vc[beta, :L], "k_idx": kic[beta, :L],
               "q": np.repeat(q[beta][None], L, 0), "q_idx": np.repeat(qi[beta][None], L, 0)}
        s2, o2, l2 = o.prefill_rows(inp, np.array([L - 1]), B_k, k)
        assert np.array_equal(sel[beta], s2[0])
        assert np.max(np.abs(out[beta] - o2[0])) < 1e-13
        assert np.max(np.abs(lse[beta] - l2[0])) < 1e-13


def check_varlen_matches_dense_per_sequence(o):
    """A packed batch: each sequence's selection and attention equal the dense brute force run on that
    sequence alone (tokens of other sequences are invisible, block indices restart at each sequence)."""
    lens = [1, 5, 16, 37, 64, 130]
    H_q, H_kv, d_h, d_idx, B_k, k = 4, 2, 8, 8, 16, 3
    cu = np.concatenate([[0], np.cumsum(lens)])
    T = int(cu[-1])
    inp = _attn_inputs(T, H_q, H_kv, d_h, d_idx, 9)
    rows = np.arange(T)
    sel, out, lse = o.prefill_varlen_rows(inp, cu, rows, B_k, k)
    for s in range(len(lens)):
        lo, hi = int(cu[s]), int(cu[s + 1])
        n = hi - lo
        part = {name: inp[name][lo:hi] for name in inp}
        want_sel = ref.dense_selection(part["q_idx"], part["k_idx"], B_k, k)
        got_sel = np.ascontiguousarray(sel[lo:hi].transpose(1, 0, 2))
        assert np.array_equal(got_sel, want_sel), s
        want, want_lse = ref.masked_attention(part["q"], part["k"], part["v"], ref.selection_mask(want_sel, n, B_k))
        assert np.max(np.abs(out[lo:hi] - want)) < 1e-12, s
        assert np.max(np.abs(lse[lo:hi] - want_lse)) < 1e-12, s


def check_varlen_cached_prefix_matches_dense(o):
    """Queries that continue a cached prefix: each sequence's chunk rows equal the dense brute force of
    the whole sequence at those positions (prefix tokens are keys only, never queried)."""
    lens_k = [48, 80, 130, 64]
    prefix = [32, 0, 64, 48]  # whole blocks of B_k = 16
    H_q, H_kv, d_h, d_idx, B_k, k = 4, 2, 8, 8, 16, 3
    cuk = np.concatenate([[0], np.cumsum(lens_k)])
    lens_q = [a - b for a, b in zip(lens_k, prefix)]
    cu = np.concatenate([[0], np.cumsum(lens_q)])
    full = _attn_inputs(int(cuk[-1]), H_q, H_kv, d_h, d_idx, 21)
    take = np.concatenate([np.arange(cuk[s] + prefix[s], cuk[s + 1]) for s in range(len(lens_k))])
    inp = {"k": full["k"], "v": full["v"], "k_idx": full["k_idx"], "q": full["q"][take], "q_idx": full["q_idx"][take]}
    sel, out, lse = o.prefill_varlen_rows(inp, cu, np.arange(int(cu[-1])), B_k, k, cu_seqlens_k=cuk)
    for s in range(len(lens_k)):
        klo, khi = int(cuk[s]), int(cuk[s + 1])
        n = khi - klo
        part = {name: full[name][klo:khi] for name in full}
        want_sel = ref.dense_selection(part["q_idx"], part["k_idx"], B_k, k)[:, prefix[s]:]
        lo, hi = int(cu[s]), int(cu[s + 1])
        assert np.array_equal(np.ascontiguousarray(sel[lo:hi].transpose(1, 0, 2)), want_sel), s
        all_sel = ref.dense_selection(part["q_idx"], part["k_idx"], B_k, k)
        want, want_lse = ref.masked_attention(part["q"], part["k"], part["v"], ref.selection_mask(all_sel, n, B_k))
        assert np.max(np.abs(out[lo:hi] - want[prefix[s]:])) < 1e-12, s
        assert np.max(np.abs(lse[lo:hi] - want_lse[prefix[s]:])) < 1e-12, s


# ------------------------------------------------------------------------------------ backward

def _bwd_case(o, N, H_q, H_kv, d_h, d_idx, B_k, k, seed):
    inp = _attn_inputs(N, H_q, H_kv, d_h, d_idx, seed)
    inp["dout"] = normal_bf16((N, H_q, d_h), seed, "ado")
    sel = o.select_rows(inp["q_idx"], inp["k_idx"], np.arange(N), B_k, k)  # [N, H_kv, k]
    nb = (N + B_k - 1) // B_k
    pairs = [(r, b) for r in range(H_kv) for b in range(nb)]
    return inp, sel, pairs, nb


def _blocks_to_tokens(g, H_kv, nb, B_k, N):
    """[(r, b) pairs in r-major order, B_k, d] -> [N, H_kv, d]."""
    d = g.shape[-1]
    return g.reshape(H_kv, nb * B_k, d)[:, :N].transpose(1, 0, 2)


BWD_SHAPES = [(96, 4, 2, 16, 8, 16, 3), (70, 2, 1, 8, 8, 8, 4), (64, 4, 2, 16, 8, 16, 4)]  # last: k*B_k >= N


def check_backward_autograd(o):
    """Main-branch dq, dk, dv equal autograd of masked dense attention under the selection mask."""
    for (N, H_q, H_kv, d_h, d_idx, B_k, k) in BWD_SHAPES:
        inp, sel, pairs, nb = _bwd_case(o, N, H_q, H_kv, d_h, d_idx, B_k, k, N + 11)
        dq = o.backward_dq_rows(inp["q"], inp["dout"], inp["k"], inp["v"], np.arange(N), sel, B_k)
        dk, dv = o.backward_dkv_blocks(inp["q"], inp["dout"], inp["k"], inp["v"], sel, pairs, B_k)
        allowed = ref.selection_mask(np.ascontiguousarray(sel.transpose(1, 0, 2)), N, B_k)
        wq, wk, wv = ref_autograd.attention_grads(inp["q"], inp["k"], inp["v"], inp["dout"], allowed)
        assert np.max(np.abs(dq - wq)) < 1e-10, np.max(np.abs(dq - wq))
        assert np.max(np.abs(_blocks_to_tokens(dk, H_kv, nb, B_k, N) - wk)) < 1e-10
        assert np.max(np.abs(_blocks_to_tokens(dv, H_kv, nb, B_k, N) - wv)) < 1e-10
        pad = nb * B_k - N
        if pad:
            assert not np.any(dk.reshape(H_kv, nb * B_k, -1)[:, N:]) and not np.any(dv.reshape(H_kv, nb * B_k, -1)[:, N:])


def check_backward_identical_keys(o):
    """All keys equal: every logit of a row is the same constant direction, so the softmax Jacobian
    annihilates dq (sum_j ds_j = 0) while dv is the mean of dout over the rows that see each key."""
    N, H_q, H_kv, d_h, d_idx, B_k, k = 80, 4, 2, 8, 8, 16, 3
    inp, sel, pairs, nb = _bwd_case(o, N, H_q, H_kv, d_h, d_idx, B_k, k, 21)
    inp["k"] = np.broadcast_to(inp["k"][:1], inp["k"].shape).copy()
    dq = o.backward_dq_rows(inp["q"], inp["dout"], inp["k"], inp["v"], np.arange(N), sel, B_k)
    assert np.max(np.abs(dq)) < 1e-12
    _, dv = o.backward_dkv_blocks(inp["q"], inp["dout"], inp["k"], inp["v"], sel, pairs, B_k)
    dv = _blocks_to_tokens(dv, H_kv, nb, B_k, N)
    allowed = ref.selection_mask(np.ascontiguousarray(sel.transpose(1, 0, 2)), N, B_k)
    dO = bf16_bits_to_f64(inp["dout"])
    G = H_q // H_kv
    for r in range(H_kv):
        wts = allowed[r] / allowed[r].sum(axis=1, keepdims=True)  # uniform weights over T(i, r)
        want = wts.T @ dO[:, r * G:(r + 1) * G, :].sum(axis=1)
        assert np.max(np.abs(dv[:, r] - want)) < 1e-12


def check_backward_dv_sums_to_dout(o):
    """Attention weights of a row sum to one, so sum_j dv[j, r] = sum_i sum_{h in r} dout[i, h]."""
    N, H_q, H_kv, d_h, d_idx, B_k, k = 150, 4, 2, 8, 8, 16, 4
    inp, sel, pairs, nb = _bwd_case(o, N, H_q, H_kv, d_h, d_idx, B_k, k, 22)
    _, dv = o.backward_dkv_blocks(inp["q"], inp["dout"], inp["k"], inp["v"], sel, pairs, B_k)
    dv = _blocks_to_tokens(dv, H_kv, nb, B_k, N)
    dO = bf16_bits_to_f64(inp["dout"])
    G = H_q // H_kv
    for r in range(H_kv):
        assert np.max(np.abs(dv[:, r].sum(axis=0) - dO[:, r * G:(r + 1) * G].sum(axis=(0, 1)))) < 1e-10


def check_kl_autograd(o):
    """Index-branch KL per (row, group) and its gradients equal autograd of the KL loss (teacher
    detached), with the loss weight 1/(N * H_kv) of the mean."""
    for (N, H_q, H_kv, d_h, d_idx, B_k, k) in BWD_SHAPES:
        inp, sel, pairs, nb = _bwd_case(o, N, H_q, H_kv, d_h, d_idx, B_k, k, N + 12)
        inp["q_idx"] = normal_bf16(inp["q_idx"].shape, N, "klq")  # non-integer index scores
        inp["k_idx"] = normal_bf16(inp["k_idx"].shape, N, "klk")
        sel = o.select_rows(inp["q_idx"], inp["k_idx"], np.arange(N), B_k, k)
        w = 1.0 / (N * H_kv)
        kl, dqi = o.kl_rows(inp["q"], inp["q_idx"], inp["k"], inp["k_idx"], np.arange(N), sel, B_k, w)
        dki = o.kl_dk_idx_blocks(inp["q"], inp["q_idx"], inp["k"], inp["k_idx"], sel, pairs, B_k, w)
        allowed = ref.selection_mask(np.ascontiguousarray(sel.transpose(1, 0, 2)), N, B_k)
        wkl, wq, wk = ref_autograd.kl_loss_grads(inp["q"], inp["k"], inp["q_idx"], inp["k_idx"], allowed, w)
        assert np.max(np.abs(kl - wkl)) < 1e-10, np.max(np.abs(kl - wkl))
        assert np.all(kl > -1e-12)  # Gibbs' inequality
        assert np.max(np.abs(dqi - wq)) < 1e-12, np.max(np.abs(dqi - wq))
        assert np.max(np.abs(_blocks_to_tokens(dki, H_kv, nb, B_k, N) - wk)) < 1e-12


def check_kl_uniform_teacher_closed_form(o):
    """q == 0 makes the teacher uniform over T, so KL(U || softmax(s)) = logsumexp(s) - mean(s) - log|T|
    and dKL/ds = softmax(s) - 1/|T|; with q_idx == 0 as well the KL and its gradients vanish."""
    N, H_q, H_kv, d_h, d_idx, B_k, k = 72, 4, 2, 8, 8, 8, 3
    inp, sel, pairs, nb = _bwd_case(o, N, H_q, H_kv, d_h, d_idx, B_k, k, 23)
    inp["q"] = np.zeros_like(inp["q"])
    kl, dqi = o.kl_rows(inp["q"], inp["q_idx"], inp["k"], inp["k_idx"], np.arange(N), sel, B_k)
    Qi, Ki = bf16_bits_to_f64(inp["q_idx"]), bf16_bits_to_f64(inp["k_idx"])
    for i in range(0, N, 7):
        for r in range(H_kv):
            toks = [j for b in sel[i, r] if b >= 0 for j in range(b * B_k, min((b + 1) * B_k, i + 1))]
            s = Ki[toks, r] @ Qi[i, r]
            lse = s.max() + math.log(np.exp(s - s.max()).sum())
            assert abs(kl[i, r] - (lse - s.mean() - math.log(len(toks)))) < 1e-10
            g = np.exp(s - lse) - 1.0 / len(toks)
            assert np.max(np.abs(dqi[i, r] - g @ Ki[toks, r])) < 1e-10
    inp["q_idx"] = np.zeros_like(inp["q_idx"])
    kl, dqi = o.kl_rows(inp["q"], inp["q_idx"], inp["k"], inp["k_idx"], np.arange(N), sel, B_k)
    dki = o.kl_dk_idx_blocks(inp["q"], inp["q_idx"], inp["k"], inp["k_idx"], sel, pairs, B_k)
    assert np.max(np.abs(kl)) < 1e-14 and np.max(np.abs(dqi)) < 1e-14 and np.max(np.abs(dki)) < 1e-14


# ------------------------------------------------------------------------------- FP8 (E4M3)

def check_e4m3_codec_closed_form(o):
    """E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, subnormals, no infinities, 448 the
    largest finite, S.1111.111 NaN): values from the format's definition, round trip of every finite
    code, ties to the even mantissa, saturation."""
    pos = [o.e4m3_decode(c) for c in range(0x7F)]
    assert pos[0] == 0.0 and pos[1] == 2.0 ** -9 and pos[7] == 7 * 2.0 ** -9     # subnormals m * 2^-9
    assert pos[8] == 2.0 ** -6 and pos[0x7E] == 448.0 == 1.75 * 2 ** 8           # smallest normal, largest
    assert all(b > a for a, b in zip(pos, pos[1:]))                               # increasing
    assert math.isnan(o.e4m3_decode(0x7F)) and math.isnan(o.e4m3_decode(0xFF))
    for c in list(range(0x7F)) + list(range(0x80, 0xFF)):
        assert o.e4m3_decode(c) == (-1.0 if c & 0x80 else 1.0) * pos[c & 0x7F]
        assert o.e4m3_encode(o.e4m3_decode(c)) == c, hex(c)
    # hand-worked: 0.1 lies in [2^-4, 2^-3), step 2^-7, 0.1 / 2^-7 = 12.8 -> 13 * 2^-7 = 1.625 * 2^-4:
    # exponent field 3, mantissa 5 -> 0x1D; 3 = 1.5 * 2^1 -> 0x44; 300 in [256, 512), step 32: 288 is
    # nearer than 320 -> 1.125 * 2^8 -> 0x79; 2^-10 is halfway between 0 and 2^-9 -> the even code 0x00
    assert o.e4m3_encode(0.1) == 0x1D and o.e4m3_decode(0x1D) == 0.1015625
    assert o.e4m3_encode(3.0) == 0x44 and o.e4m3_encode(-3.0) == 0xC4
    assert o.e4m3_encode(300.0) == 0x79 and o.e4m3_decode(0x79) == 288.0
    assert o.e4m3_encode(2.0 ** -10) == 0x00 and o.e4m3_encode(3 * 2.0 ** -10) == 0x02   # 1.5 -> 2 (even)
    assert o.e4m3_encode(1e9) == 0x7E and o.e4m3_encode(-1e9) == 0xFE and o.e4m3_encode(-0.0) == 0x80
    for c in range(0x08, 0x7E):                                                   # midpoints of normals
        mid = 0.5 * (pos[c] + pos[c + 1])
        assert o.e4m3_encode(mid) == (c if c % 2 == 0 else c + 1), hex(c)


def check_e4m3_quantize_rows(o):
    """Per-row scale amax / 448: each row's largest magnitude becomes +-448, and every value is
    within half a step of the format (relative 2^-4 in the normal range) after dequantisation."""
    x = normal_bf16((50, 4, 32), 31, "e4m3")
    codes, scales = o.quantize_e4m3(x)
    X = bf16_bits_to_f64(x)
    amax = np.abs(X).max(axis=-1)
    assert np.array_equal(scales, amax / 448.0)
    deq = np.vectorize(o.e4m3_decode)(codes) * scales[..., None]
    top = np.abs(X) == amax[..., None]
    assert np.all(np.abs(codes[top] & 0x7F) == 0x7E)
    rel = np.abs(X) / scales[..., None]
    normal = rel >= 2.0 ** -6
    assert np.all(np.abs(deq - X)[normal] <= 2.0 ** -4 * np.abs(X)[normal])
    assert np.all(np.abs(deq - X)[~normal] <= 2.0 ** -10 * np.broadcast_to(scales[..., None], X.shape)[~normal])


def _e4m3_case(o, N, H_q, H_kv, d_h, seed):
    inp = _attn_inputs(N, H_q, H_kv, d_h, 8, seed)
    q8, k8, v8 = (o.quantize_e4m3(inp[n]) for n in ("q", "k", "v"))
    dec = np.vectorize(o.e4m3_decode)
    deq = [dec(c) * s[..., None] for c, s in (q8, k8, v8)]
    return inp, (q8, k8, v8), deq


def check_attention_e4m3_dense_invariant(o):
    """FP8 main branch with k*B_k >= N: textbook dense causal GQA attention on the dequantised q, k, v."""
    N, H_q, H_kv, d_h, B_k, k = 80, 4, 2, 16, 16, 5
    inp, (q8, k8, v8), (Q, K, V) = _e4m3_case(o, N, H_q, H_kv, d_h, 41)
    rows = np.arange(N)
    sel = o.select_rows(inp["q_idx"], inp["k_idx"], rows, B_k, k)
    out, lse = o.attend_rows_e4m3(q8, k8, v8, rows, sel, B_k)
    want, want_lse = ref.dense_causal_gqa_f64(Q, K, V)
    assert np.max(np.abs(out - want)) < 1e-12 and np.max(np.abs(lse - want_lse)) < 1e-12


def check_attention_e4m3_masked_bruteforce(o):
    """FP8 main branch with k*B_k < N: dense attention under the selection mask on the dequantised values."""
    N, H_q, H_kv, d_h, B_k, k = 150, 4, 2, 16, 16, 3
    inp, (q8, k8, v8), (Q, K, V) = _e4m3_case(o, N, H_q, H_kv, d_h, 42)
    rows = np.arange(N)
    sel = o.select_rows(inp["q_idx"], inp["k_idx"], rows, B_k, k)
    out, lse = o.attend_rows_e4m3(q8, k8, v8, rows, sel, B_k)
    allowed = ref.selection_mask(np.ascontiguousarray(sel.transpose(1, 0, 2)), N, B_k)
    want, want_lse = ref.masked_attention_f64(Q, K, V, allowed)
    assert np.max(np.abs(out - want)) < 1e-12 and np.max(np.abs(lse - want_lse)) < 1e-12


ALL_CHECKS = [
    check_selection_bruteforce,
    check_selection_ties_closed_form,
    check_selection_planted_winners,
    check_selection_invariants,
    check_attention_dense_invariant,
    check_attention_masked_bruteforce,
    check_attention_zero_keys,
    check_attention_k1_block_local,
    check_attention_hand_example,
    check_combine_identity,
    check_kv2q_bruteforce,
    check_decode_matches_prefill_row,
    check_varlen_matches_dense_per_sequence,
    check_varlen_cached_prefix_matches_dense,
    check_backward_autograd,
    check_backward_identical_keys,
    check_backward_dv_sums_to_dout,
    check_kl_autograd,
    check_kl_uniform_teacher_closed_form,
    check_e4m3_codec_closed_form,
    check_e4m3_quantize_rows,
    check_attention_e4m3_dense_invariant,
    check_attention_e4m3_masked_bruteforce,
]
