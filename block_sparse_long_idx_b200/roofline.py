"""Analytic work of the MSA forward path, used for roofline fractions.

FLOP model ("MiniMax Sparse Attention" explainer, section 04; abstract): causal dense GQA costs
2*H_q*d_h*N^2, the MSA main branch 4*H_q*d_h*N*k*B_k (two matmuls of 2*d_h FLOP per query-head and
attended token, k*B_k tokens per query), and the index branch H_kv*d_idx*N^2 (one 2*d_idx dot product
per query, visible key and group, about N^2/2 visible pairs).

Byte models are the algorithmic minimum traffic of each HBM-bound kernel in this implementation's
data layout (bf16 tensors, fp32 lse, bf16 normalised partials + fp32 partial lse).
"""
from __future__ import annotations


def gqa_flops(N: int, H_q: int, d_h: int) -> float:
    return 2.0 * H_q * d_h * N * N


def main_branch_flops(N: int, H_q: int, d_h: int, k: int, B_k: int) -> float:
    return 4.0 * H_q * d_h * N * k * B_k


def main_branch_backward_flops(N: int, H_q: int, d_h: int, k: int, B_k: int) -> float:
    """Backward of the main branch with the selections fixed: per (row, head, selected block) five
    B_k x d_h products (S recomputed, dP = dO V^T, dV += P^T dO, dK += dS^T Q, dQ += dS K), 2.5x the
    forward's two."""
    return 10.0 * H_q * d_h * N * k * B_k


def index_branch_flops(N: int, H_kv: int, d_idx: int) -> float:
    return 2.0 * H_kv * d_idx * N * N / 2.0


def msa_flops(N, H_q, H_kv, d_h, d_idx, k, B_k) -> float:
    return main_branch_flops(N, H_q, d_h, k, B_k) + index_branch_flops(N, H_kv, d_idx)


def n_selected(N: int, k: int, B_k: int) -> int:
    """Total number of selected (row, block) pairs per group: sum_i min(k, floor(i/B_k) + 1)."""
    total = 0
    nb = (N + B_k - 1) // B_k
    for t in range(nb):
        rows = min(B_k, N - t * B_k)
        total += rows * min(k, t + 1)
    return total


def combine_bytes(N: int, H_q: int, H_kv: int, d_h: int, k: int, B_k: int) -> float:
    """Stage-2 merge: read every valid partial (bf16 output + fp32 lse), write bf16 out + fp32 lse."""
    pairs = n_selected(N, k, B_k) * (H_q // H_kv) * H_kv  # (row, head, slot) triples
    return pairs * (2 * d_h + 4) + N * H_q * (2 * d_h + 4)


def attn_min_bytes(N: int, H_q: int, H_kv: int, d_h: int, k: int, B_k: int) -> float:
    """Stage-1 minimum HBM traffic: q, k, v read once, every partial written once."""
    pairs = n_selected(N, k, B_k) * H_q
    return 2 * N * H_q * d_h + 2 * 2 * N * H_kv * d_h + pairs * (2 * d_h + 4)


def decode_bytes(lens, H_q: int, H_kv: int, d_h: int, d_idx: int, k: int, B_k: int) -> dict:
    """Decode kernels' algorithmic bytes: pooled index scan of the visible non-local cache blocks, and
    the selected K/V blocks (the local block only up to the query)."""
    pool = 0
    attn = 0
    for L in lens:
        L = int(L)
        loc = (L - 1) // B_k
        pool += loc * B_k * H_kv * d_idx * 2
        n_full = min(k - 1, loc)
        toks = n_full * B_k + (L - loc * B_k)
        attn += H_kv * toks * d_h * 2 * 2
    return {"dec_pool": float(pool), "dec_attn": float(attn)}


def kv2q_bytes(N: int, H_kv: int, k: int, B_k: int, window: int = 2048) -> float:
    """KV->Q inversion (counting sort per query window): the selections are read twice (the count
    pass and the scatter pass, 4 B per (group, row, slot)), every valid entry is written once (4 B),
    and the per-(group, block, window) counts, bases and item counts are written and read once
    (3 x 4 B each)."""
    nb = (N + B_k - 1) // B_k
    n_windows = (N + window - 1) // window
    slots = H_kv * N * k
    valid = n_selected(N, k, B_k) * H_kv
    return 8.0 * slots + 4.0 * valid + 12.0 * H_kv * nb * n_windows


def quant_bytes(N: int, H: int, d: int, B_k: int = 128) -> float:
    """E4M3 quantisation of one [N, H, d] bf16 tensor: read 2 B and write a 1-byte code per element, write
    the scale and its reciprocal (4 B each) per row of the padded token range and the block maxima."""
    S = (N + B_k - 1) // B_k * B_k
    return 3.0 * N * H * d + 8.0 * S * H + 4.0 * H * (S // B_k)
