"""Gradients by automatic differentiation, used to pin the oracle's hand-derived backward.

The forward definitions here are the textbook ones (masked dense softmax attention, the KL
alignment loss between the index branch's softmax and the group-averaged attention weights) written
with plain PyTorch CPU ops in float64; torch.autograd differentiates them. Nothing here is shared
with the oracle (which applies the softmax Jacobian by hand, row by row) or with the CUDA library.
"""
from __future__ import annotations

import numpy as np
import torch

from block_sparse_long_idx_b200.synth import bf16_bits_to_f64


def _t(a, grad=False):
    return torch.tensor(bf16_bits_to_f64(a), dtype=torch.float64, requires_grad=grad)


def attention_grads(q, kk, v, dout, allowed):
    """d/d(q, k, v) of sum(dout * out) for attention under the mask allowed[r, i, j].

    q, dout [N, H_q, d_h]; kk, v [N, H_kv, d_h] (bf16 bits). Returns float64 numpy (dq, dk, dv)."""
    Q, K, V = _t(q, True), _t(kk, True), _t(v, True)
    dO = _t(dout)
    N, H_q, d_h = Q.shape
    H_kv = K.shape[1]
    G = H_q // H_kv
    M = torch.tensor(allowed)
    loss = torch.zeros((), dtype=torch.float64)
    for h in range(H_q):
        r = h // G
        S = (Q[:, h, :] @ K[:, r, :].T) / np.sqrt(d_h)
        S = S.masked_fill(~M[r], float("-inf"))
        out = torch.softmax(S, dim=1) @ V[:, r, :]
        loss = loss + (out * dO[:, h, :]).sum()
    loss.backward()
    return Q.grad.numpy(), K.grad.numpy(), V.grad.numpy()


def kl_loss_grads(q, kk, q_idx, k_idx, allowed, w: float = 1.0):
    """KL alignment of the index branch: for every row i and group r over the allowed tokens,
    KL(P || P_idx) with P the mean over the group's heads of the attention weights (held constant)
    and P_idx the softmax of the unscaled index scores. Returns (kl [N, H_kv], d q_idx, d k_idx) of
    w * sum(kl), float64 numpy."""
    Q, K = _t(q), _t(kk)
    QI, KI = _t(q_idx, True), _t(k_idx, True)
    N, H_q, d_h = Q.shape
    H_kv = K.shape[1]
    G = H_q // H_kv
    M = torch.tensor(allowed)
    kl = torch.zeros((N, H_kv), dtype=torch.float64)
    rows = []
    for r in range(H_kv):
        with torch.no_grad():
            P = torch.zeros((N, N), dtype=torch.float64)
            for h in range(r * G, (r + 1) * G):
                S = (Q[:, h, :] @ K[:, r, :].T) / np.sqrt(d_h)
                P = P + torch.softmax(S.masked_fill(~M[r], float("-inf")), dim=1) / G
        Si = (QI[:, r, :] @ KI[:, r, :].T).masked_fill(~M[r], float("-inf"))
        logq = torch.log_softmax(Si, dim=1)
        logP = torch.log(torch.where(M[r], P, torch.ones_like(P)))
        terms = torch.where(M[r], P * (logP - logq), torch.zeros_like(P))
        rows.append(terms.sum(dim=1))
    kl = torch.stack(rows, dim=1)
    (w * kl.sum()).backward()
    return kl.detach().numpy(), QI.grad.numpy(), KI.grad.numpy()
