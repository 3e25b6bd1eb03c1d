"""Independent dense brute force used to pin the C oracle on tiny inputs.

Different algorithms from the oracle on purpose: the whole N x N score matrix is built with one
matrix product, pooled with a reshape-max, ranked with numpy's lexsort; attention is the
textbook dense causal GQA softmax with a mask matrix. Shares no code with the oracle or the
CUDA library.
"""
from __future__ import annotations

import numpy as np

from block_sparse_long_idx_b200.synth import bf16_bits_to_f64


def dense_selection(q_idx, k_idx, B_k: int, k: int) -> np.ndarray:
    """Brute-force Top-k block selection, [H_kv, N, k] int32 (ascending, -1 padded)."""
    N, H_kv, _ = k_idx.shape
    nb = (N + B_k - 1) // B_k
    Q = bf16_bits_to_f64(q_idx)
    K = bf16_bits_to_f64(k_idx)
    out = np.full((H_kv, N, k), -1, dtype=np.int32)
    causal = np.tril(np.ones((N, N), dtype=bool))
    for r in range(H_kv):
        S = Q[:, r, :] @ K[:, r, :].T
        S = np.where(causal, S, -np.inf)
        Sp = np.full((N, nb * B_k), -np.inf)
        Sp[:, :N] = S
        pooled = Sp.reshape(N, nb, B_k).max(axis=2)
        for i in range(N):
            loc = i // B_k
            cand = np.arange(loc)
            order = np.lexsort((cand, -pooled[i, cand]))  # primary: score desc, secondary: block asc
            chosen = sorted(list(cand[order[: k - 1]]) + [loc])
            out[r, i, : len(chosen)] = chosen
    return out


def dense_causal_gqa(q, kk, v):
    """Dense causal GQA attention in float64. Returns (out [N, H_q, d_h], lse [N, H_q])."""
    return dense_causal_gqa_f64(bf16_bits_to_f64(q), bf16_bits_to_f64(kk), bf16_bits_to_f64(v))


def dense_causal_gqa_f64(Q, K, V):
    """dense_causal_gqa on float64 arrays."""
    N, H_q, d_h = Q.shape
    H_kv = K.shape[1]
    G = H_q // H_kv
    mask = np.tril(np.ones((N, N), dtype=bool))
    out = np.zeros((N, H_q, d_h))
    lse = np.zeros((N, H_q))
    for h in range(H_q):
        r = h // G
        S = (Q[:, h, :] @ K[:, r, :].T) / np.sqrt(d_h)
        S = np.where(mask, S, -np.inf)
        m = S.max(axis=1, keepdims=True)
        P = np.exp(S - m)
        Z = P.sum(axis=1, keepdims=True)
        out[:, h, :] = (P / Z) @ V[:, r, :]
        lse[:, h] = (m + np.log(Z))[:, 0]
    return out, lse


def masked_attention(q, kk, v, allowed):
    """Attention with an explicit boolean mask allowed[h_group, i, j]. float64."""
    return masked_attention_f64(bf16_bits_to_f64(q), bf16_bits_to_f64(kk), bf16_bits_to_f64(v), allowed)


def masked_attention_f64(Q, K, V, allowed):
    """masked_attention on float64 arrays."""
    N, H_q, d_h = Q.shape
    H_kv = K.shape[1]
    G = H_q // H_kv
    out = np.zeros((N, H_q, d_h))
    lse = np.zeros((N, H_q))
    for h in range(H_q):
        r = h // G
        S = (Q[:, h, :] @ K[:, r, :].T) / np.sqrt(d_h)
        S = np.where(allowed[r], S, -np.inf)
        m = S.max(axis=1, keepdims=True)
        P = np.exp(S - m)
        Z = P.sum(axis=1, keepdims=True)
        out[:, h, :] = (P / Z) @ V[:, r, :]
        lse[:, h] = (m + np.log(Z))[:, 0]
    return out, lse


def selection_mask(sel, N: int, B_k: int) -> np.ndarray:
    """allowed[r, i, j] = (j <= i) and block(j) in sel[r, i]."""
    H_kv = sel.shape[0]
    allowed = np.zeros((H_kv, N, N), dtype=bool)
    blk = np.arange(N) // B_k
    for r in range(H_kv):
        for i in range(N):
            chosen = [b for b in sel[r, i] if b >= 0]
            allowed[r, i] = np.isin(blk, chosen) & (np.arange(N) <= i)
    return allowed


def brute_kv2q(block_idx, B_k: int):
    """For each (r, b): rows i ascending with b in sel[r, i], as i*k + slot."""
    H_kv, N, k = block_idx.shape
    nb = (N + B_k - 1) // B_k
    lists = []
    for r in range(H_kv):
        per_b = []
        for b in range(nb):
            hits = np.argwhere(block_idx[r] == b)  # rows ascending (argwhere is row-major)
            per_b.append((hits[:, 0] * k + hits[:, 1]).astype(np.int32))
        lists.append(per_b)
    return lists
