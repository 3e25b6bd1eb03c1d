"""Seeded synthetic inputs for the MSA forward path.

This module only draws random numbers and rounds them to bf16 bit patterns.
It holds none of the method's arithmetic (no scoring, pooling, selection,
softmax or merging), so that both the CPU oracle and the CUDA path can take
their inputs from it without sharing any of the method's code.

Workloads (MiniMax Sparse Attention explainer, sections 04-06, and the paper
abstract): GQA heads H_q = 64 / H_kv = 4, head dim 128, KV blocks of
B_k = 128 tokens, k = 16 selected blocks per (query, group).

Value recipes:
  * q, k, v: N(0, 1) samples rounded to bf16 (round to nearest even).
  * q_idx, k_idx: integers drawn uniformly from {-3, ..., 3}, stored as bf16
    (exact), so every index score is an exactly representable integer.
  * planted (the 128K workload): per group r a direction u[r] ~ N(0, I); 32
    distinct "needle" blocks get k_idx += 2*sign(u[r]) on all their tokens;
    each query row gets q_idx += sign(u[r]) with probability 1/4 per (i, r).
    Values stay within [-5, 5], still exact in bf16.
  * decode: per-sequence cache lengths uniform on [16384, 131072].

Every array is generated in fixed chunks of 2**22 elements, each chunk from its
own PCG64 stream keyed by (seed, tensor name, chunk), so results do not depend
on the number of worker threads.
"""
from __future__ import annotations

import hashlib
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace

import numpy as np

CHUNK = 1 << 22


# --------------------------------------------------------------------------
# bf16 bit-pattern helpers (storage format only)
# --------------------------------------------------------------------------
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 with round-to-nearest-even; returns uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(b).astype(np.float64)


# --------------------------------------------------------------------------
# chunked deterministic generation
# --------------------------------------------------------------------------
def _stream_key(name: str) -> int:
    return int.from_bytes(hashlib.sha256(name.encode()).digest()[:4], "little")


def _rng(seed: int, name: str, chunk: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, _stream_key(name), chunk])))


def _workers() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _fill_chunks(n: int, fn) -> None:
    nchunks = (n + CHUNK - 1) // CHUNK
    if nchunks <= 1:
        for c in range(nchunks):
            fn(c, 0, n)
        return
    with ThreadPoolExecutor(_workers()) as ex:
        list(ex.map(lambda c: fn(c, c * CHUNK, min(n, (c + 1) * CHUNK)), range(nchunks)))


def normal_bf16(shape, seed: int, name: str) -> np.ndarray:
    """N(0,1) draws rounded to bf16 bits."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)

    def fn(c, lo, hi):
        x = _rng(seed, name, c).standard_normal(hi - lo, dtype=np.float32)
        out[lo:hi] = f32_to_bf16_bits(x)

    _fill_chunks(n, fn)
    return out.reshape(shape)


def int_uniform_bf16(shape, lo_v: int, hi_v: int, seed: int, name: str) -> np.ndarray:
    """Integers uniform on {lo_v, ..., hi_v} stored as bf16 bits (exact for |v| <= 256)."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)

    def fn(c, lo, hi):
        x = _rng(seed, name, c).integers(lo_v, hi_v + 1, size=hi - lo, dtype=np.int8)
        out[lo:hi] = f32_to_bf16_bits(x.astype(np.float32))

    _fill_chunks(n, fn)
    return out.reshape(shape)


# --------------------------------------------------------------------------
# workload configurations
# --------------------------------------------------------------------------
@dataclass(frozen=True)
class PrefillConfig:
    name: str
    N: int
    H_q: int
    H_kv: int
    d_h: int
    d_idx: int
    B_k: int
    k: int
    seed: int
    planted: bool = False
    n_needles: int = 32

    @property
    def G(self) -> int:
        return self.H_q // self.H_kv

    @property
    def nb(self) -> int:
        return (self.N + self.B_k - 1) // self.B_k

    def with_(self, **kw) -> "PrefillConfig":
        return replace(self, **kw)


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    B: int
    L_max: int
    len_lo: int
    len_hi: int
    H_q: int
    H_kv: int
    d_h: int
    d_idx: int
    B_k: int
    k: int
    seed: int

    @property
    def G(self) -> int:
        return self.H_q // self.H_kv

    def with_(self, **kw) -> "DecodeConfig":
        return replace(self, **kw)


TINY = PrefillConfig("tiny_prefill_N2048", N=2048, H_q=8, H_kv=2, d_h=64, d_idx=32, B_k=128, k=4, seed=0)
P32K = PrefillConfig("prefill_N32768", N=32768, H_q=64, H_kv=4, d_h=128, d_idx=64, B_k=128, k=16, seed=1)
P128K = PrefillConfig("planted_prefill_N131072", N=131072, H_q=64, H_kv=4, d_h=128, d_idx=64, B_k=128, k=16,
                      seed=2, planted=True)
P1M = PrefillConfig("prefill_N1048576", N=1048576, H_q=64, H_kv=4, d_h=128, d_idx=64, B_k=128, k=16, seed=3)
DECODE64 = DecodeConfig("decode_B64_L16K-128K", B=64, L_max=131072, len_lo=16384, len_hi=131072, H_q=64, H_kv=4,
                        d_h=128, d_idx=64, B_k=128, k=16, seed=4)
# the same decode step over shorter caches (2 GB of K/V): small enough for detailed profiler captures
DECODE64_SHORT = DecodeConfig("decode_B64_L2K-16K", B=64, L_max=16384, len_lo=2048, len_hi=16384, H_q=64, H_kv=4,
                              d_h=128, d_idx=64, B_k=128, k=16, seed=5)

@dataclass(frozen=True)
class VarlenConfig:
    """A batch of independent causal sequences packed along the token axis (cu_seqlens layout)."""
    name: str
    lens: tuple
    H_q: int
    H_kv: int
    d_h: int
    d_idx: int
    B_k: int
    k: int
    seed: int
    prefix: tuple = ()  # per sequence, tokens already in the key cache before its query rows (whole blocks)

    @property
    def T(self) -> int:
        return int(sum(self.lens))

    def prefixes(self) -> np.ndarray:
        return np.asarray(self.prefix if self.prefix else (0,) * len(self.lens), dtype=np.int64)

    @property
    def Tk(self) -> int:
        return int(self.T + self.prefixes().sum())

    def cu_seqlens(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.lens)]).astype(np.int32)

    def cu_seqlens_k(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(np.asarray(self.lens) + self.prefixes())]).astype(np.int32)

    def packed(self) -> "PrefillConfig":
        """The key-side tensors: all tokens (cached prefixes and query rows) of all sequences."""
        return PrefillConfig(self.name, N=self.Tk, H_q=self.H_q, H_kv=self.H_kv, d_h=self.d_h, d_idx=self.d_idx,
                             B_k=self.B_k, k=self.k, seed=self.seed)


def varlen_lengths(n_seq: int, total: int, lo: int, seed: int) -> tuple:
    """n_seq lengths >= lo summing to total, drawn from a seeded Dirichlet-like split (long/short mix)."""
    rng = np.random.default_rng(np.random.SeedSequence([seed, 77]))
    w = rng.exponential(1.0, n_seq)
    extra = total - n_seq * lo
    lens = lo + np.floor(w / w.sum() * extra).astype(np.int64)
    lens[: total - int(lens.sum())] += 1
    return tuple(int(x) for x in lens)


# 128K tokens as 16 sequences of mixed lengths (>= 1K): the serving-form prefill of the same model shape
VARLEN128K = VarlenConfig("varlen_16seq_T131072", lens=varlen_lengths(16, 131072, 1024, 6), H_q=64, H_kv=4, d_h=128,
                          d_idx=64, B_k=128, k=16, seed=6)

PREFILL_CONFIGS = {c.name: c for c in (TINY, P32K, P128K, P1M)}
DECODE_CONFIGS = {c.name: c for c in (DECODE64, DECODE64_SHORT)}


# --------------------------------------------------------------------------
# input tensors
# --------------------------------------------------------------------------
def prefill_index_inputs(cfg: PrefillConfig) -> dict:
    """q_idx, k_idx as bf16 bits, shapes [N, H_kv, d_idx]; planting applied if cfg.planted."""
    shp = (cfg.N, cfg.H_kv, cfg.d_idx)
    q_idx = int_uniform_bf16(shp, -3, 3, cfg.seed, "q_idx")
    k_idx = int_uniform_bf16(shp, -3, 3, cfg.seed, "k_idx")
    if cfg.planted:
        q_idx, k_idx = _plant(cfg, q_idx, k_idx)
    return {"q_idx": q_idx, "k_idx": k_idx}


def planted_structure(cfg: PrefillConfig):
    """The planted recipe's random draws: sign(u[r]) [H_kv, d_idx], needle blocks [H_kv, n_needles],
    Bernoulli(1/4) row mask [N, H_kv]."""
    g = _rng(cfg.seed, "planted", 0)
    u = g.standard_normal((cfg.H_kv, cfg.d_idx))
    sgn = np.where(u >= 0, 1.0, -1.0).astype(np.float32)
    needles = np.stack([np.sort(g.choice(cfg.nb, size=cfg.n_needles, replace=False)) for _ in range(cfg.H_kv)])
    rowmask = _rng(cfg.seed, "planted_rows", 0).random((cfg.N, cfg.H_kv)) < 0.25
    return sgn, needles, rowmask


def _plant(cfg: PrefillConfig, q_idx: np.ndarray, k_idx: np.ndarray):
    sgn, needles, rowmask = planted_structure(cfg)
    qf = bf16_bits_to_f32(q_idx).reshape(cfg.N, cfg.H_kv, cfg.d_idx)
    kf = bf16_bits_to_f32(k_idx).reshape(cfg.N, cfg.H_kv, cfg.d_idx)
    for r in range(cfg.H_kv):
        for b in needles[r]:
            lo, hi = b * cfg.B_k, min(cfg.N, (b + 1) * cfg.B_k)
            kf[lo:hi, r, :] += 2.0 * sgn[r]
        qf[rowmask[:, r], r, :] += sgn[r]
    return f32_to_bf16_bits(qf), f32_to_bf16_bits(kf)


def prefill_qkv(cfg: PrefillConfig) -> dict:
    """q [N, H_q, d_h], k, v [N, H_kv, d_h] as bf16 bits."""
    return {
        "q": normal_bf16((cfg.N, cfg.H_q, cfg.d_h), cfg.seed, "q"),
        "k": normal_bf16((cfg.N, cfg.H_kv, cfg.d_h), cfg.seed, "k"),
        "v": normal_bf16((cfg.N, cfg.H_kv, cfg.d_h), cfg.seed, "v"),
    }


def prefill_inputs(cfg: PrefillConfig) -> dict:
    d = prefill_index_inputs(cfg)
    d.update(prefill_qkv(cfg))
    return d


def varlen_inputs(cfg: VarlenConfig) -> dict:
    """Packed tensors of all sequences plus cu_seqlens [B+1] (query rows) and cu_seqlens_k [B+1] (key
    rows); every sequence is an independent causal problem. k, v, k_idx hold every token of every
    sequence ([Tk, heads, dim]); q, q_idx hold each sequence's last len (query) tokens ([T, ...])."""
    d = prefill_inputs(cfg.packed())
    cu, cuk = cfg.cu_seqlens(), cfg.cu_seqlens_k()
    pre = cfg.prefixes()
    if pre.any():
        take = np.concatenate([np.arange(cuk[s] + pre[s], cuk[s + 1]) for s in range(len(cfg.lens))]).astype(np.int64)
        d["q"] = np.ascontiguousarray(d["q"][take])
        d["q_idx"] = np.ascontiguousarray(d["q_idx"][take])
    d["cu_seqlens"] = cu
    d["cu_seqlens_k"] = cuk
    return d


def decode_lens(cfg: DecodeConfig) -> np.ndarray:
    return _rng(cfg.seed, "lens", 0).integers(cfg.len_lo, cfg.len_hi + 1, size=cfg.B).astype(np.int32)


def decode_inputs(cfg: DecodeConfig, lens=None) -> dict:
    """Caches [B, L_max, H_kv, d] holding each sequence's first len tokens (the rest is zero and never
    read), one query per sequence. Each sequence's cache rows come from their own streams."""
    B, L = cfg.B, cfg.L_max
    lens = decode_lens(cfg) if lens is None else np.asarray(lens, dtype=np.int32)
    kc = np.zeros((B, L, cfg.H_kv, cfg.d_h), dtype=np.uint16)
    vc = np.zeros_like(kc)
    kic = np.zeros((B, L, cfg.H_kv, cfg.d_idx), dtype=np.uint16)
    for b in range(B):
        n = int(min(max(lens[b], 0), L))
        kc[b, :n] = normal_bf16((n, cfg.H_kv, cfg.d_h), cfg.seed, f"k_cache/{b}")
        vc[b, :n] = normal_bf16((n, cfg.H_kv, cfg.d_h), cfg.seed, f"v_cache/{b}")
        kic[b, :n] = int_uniform_bf16((n, cfg.H_kv, cfg.d_idx), -3, 3, cfg.seed, f"k_idx_cache/{b}")
    return {
        "lens": lens,
        "q": normal_bf16((B, cfg.H_q, cfg.d_h), cfg.seed, "dq"),
        "q_idx": int_uniform_bf16((B, cfg.H_kv, cfg.d_idx), -3, 3, cfg.seed, "dq_idx"),
        "k_cache": kc,
        "v_cache": vc,
        "k_idx_cache": kic,
    }


def sample_rows(N: int, B_k: int, n: int, seed: int) -> np.ndarray:
    """Sorted sample of query rows: {0, B_k-1, B_k, N-1} plus uniform draws without replacement."""
    fixed = sorted({0, min(B_k - 1, N - 1), min(B_k, N - 1), N - 1})
    if n >= N:
        return np.arange(N, dtype=np.int64)
    g = _rng(seed, "rows", 0)
    rest = g.choice(N, size=min(N, n + len(fixed)), replace=False)
    rows = list(dict.fromkeys(list(fixed) + [int(x) for x in rest]))[: max(n, len(fixed))]
    return np.array(sorted(rows), dtype=np.int64)
