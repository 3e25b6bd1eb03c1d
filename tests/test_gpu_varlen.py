"""GPU parity, packed-batch (varlen) prefill: every sequence of a cu_seqlens batch is an independent
causal problem. Selections (local block ids, bit-exact) and outputs (tolerance) against the oracle
run on each sequence alone; ragged, tiny and empty sequences; several passes; and a batch of one
sequence equal to the single-sequence entry points."""
import zlib

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import block_sparse_long_idx_b200 as msa  # noqa: E402
import oracle  # noqa: E402
from block_sparse_long_idx_b200 import synth  # noqa: E402
from tests.gpu_util import assert_lse_close, assert_out_close, assert_selection_equal, bf16_to_f64, dev  # noqa: E402

# name, lengths, H_q, H_kv, d_h, d_idx, k, check all rows
CASES = [
    ("ragged_small", (1, 5, 127, 128, 129, 300, 1000, 2049), 8, 2, 64, 32, 4, True),
    ("empty_seqs", (0, 500, 0, 0, 300, 1), 4, 1, 128, 64, 3, True),
    ("G16_mixed", (3000, 700, 5000, 1, 2500), 64, 4, 128, 64, 16, False),
    ("G1_k8", (900, 1300, 64), 2, 2, 64, 128, 8, True),
]


def _cfg(name, lens, H_q, H_kv, d_h, d_idx, k, prefix=()):
    return synth.VarlenConfig(name, lens=tuple(lens), H_q=H_q, H_kv=H_kv, d_h=d_h, d_idx=d_idx, B_k=128, k=k,
                              seed=zlib.crc32(name.encode()) % 1000, prefix=tuple(prefix))


def _run(cfg, max_rows_per_pass=0):
    inp = synth.varlen_inputs(cfg)
    t = {n: dev(inp[n]) for n in ("q", "k", "v", "q_idx", "k_idx")}
    cuk = inp["cu_seqlens_k"] if cfg.prefix else None
    out, lse, bi = msa.msa_sparse_prefill_varlen(t["q"], t["k"], t["v"], t["q_idx"], t["k_idx"], inp["cu_seqlens"],
                                                 128, cfg.k, max_rows_per_pass=max_rows_per_pass, cu_seqlens_k=cuk)
    torch.cuda.synchronize()
    return inp, out, lse, bi


def _check(cfg, rows, max_rows_per_pass=0):
    inp, out, lse, bi = _run(cfg, max_rows_per_pass)
    sel, want, want_lse = oracle.prefill_varlen_rows(inp, inp["cu_seqlens"], rows, 128, cfg.k,
                                                     cu_seqlens_k=inp["cu_seqlens_k"])
    got_sel = bi.cpu().numpy()[:, rows, :]
    assert_selection_equal(got_sel, np.ascontiguousarray(sel.transpose(1, 0, 2)), rows)
    assert_out_close(bf16_to_f64(out)[rows], want)
    assert_lse_close(lse.cpu().numpy()[rows].astype(np.float64), want_lse)


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_varlen_prefill(case):
    name, lens, H_q, H_kv, d_h, d_idx, k, full = case
    cfg = _cfg(name, lens, H_q, H_kv, d_h, d_idx, k)
    if full:
        rows = np.arange(cfg.T)
    else:  # every sequence's first, last and block-boundary rows plus a uniform sample
        cu = cfg.cu_seqlens()
        fixed = set()
        for s in range(len(lens)):
            if lens[s]:
                for r in (0, 127, 128, lens[s] - 1):
                    if r < lens[s]:
                        fixed.add(int(cu[s]) + r)
        rng = np.random.default_rng(5)
        rows = np.unique(np.concatenate([np.array(sorted(fixed)), rng.choice(cfg.T, 400, replace=False)]))
    _check(cfg, rows)


def test_varlen_multi_pass():
    """A workspace for one 2048-row window: the attention runs window by window across sequences."""
    cfg = _cfg("passes", (1500, 3000, 200, 2300), 8, 2, 64, 64, 6)
    _check(cfg, np.arange(cfg.T), max_rows_per_pass=2048)


def test_varlen_single_sequence_equals_dense_path():
    """B = 1: identical selections and outputs to msa_index_topk + msa_build_kv2q + msa_sparse_prefill."""
    cfg = _cfg("single", (3333,), 16, 2, 128, 64, 5)
    inp = synth.varlen_inputs(cfg)
    t = {n: dev(inp[n]) for n in ("q", "k", "v", "q_idx", "k_idx")}
    out_v, lse_v, bi_v = msa.msa_sparse_prefill_varlen(t["q"], t["k"], t["v"], t["q_idx"], t["k_idx"],
                                                       inp["cu_seqlens"], 128, cfg.k)
    bi = msa.msa_index_topk(t["q_idx"], t["k_idx"], 128, cfg.k)
    kv = msa.msa_build_kv2q(bi, 128)
    out, lse = msa.msa_sparse_prefill(t["q"], t["k"], t["v"], bi, kv)
    torch.cuda.synchronize()
    assert torch.equal(bi_v, bi)
    assert torch.equal(out_v, out)
    assert torch.equal(lse_v, lse)


def test_varlen_full_size_sampled():
    """The bench's packed batch (16 sequences, 131072 tokens, 64 q / 4 kv heads, d_h 128, k 16) on
    sampled rows of every sequence."""
    cfg = synth.VARLEN128K
    cu = cfg.cu_seqlens()
    rng = np.random.default_rng(11)
    picks = []
    for s in range(len(cfg.lens)):
        n = cfg.lens[s]
        local = np.unique(np.concatenate([[0, 127, 128, n - 1], rng.choice(n, 24, replace=False)]))
        picks.append(int(cu[s]) + local[local < n])
    _check(cfg, np.concatenate(picks))


CHUNKED = [
    # name, query lengths, cached prefixes, H_q, H_kv, d_h, d_idx, k, all rows
    ("chunked_mixed", (300, 1000, 1, 129, 0), (128, 0, 2048, 256, 384), 8, 2, 64, 32, 4, True),
    ("chunked_G16", (2000, 700, 1500), (4096, 1024, 0), 64, 4, 128, 64, 16, False),
]


@pytest.mark.parametrize("case", CHUNKED, ids=[c[0] for c in CHUNKED])
def test_varlen_chunked_prefill(case):
    """Queries continuing a KV cache: each sequence's keys hold a cached prefix (whole blocks) then its
    query rows, which sit at the sequence's last positions."""
    name, lens, prefix, H_q, H_kv, d_h, d_idx, k, full = case
    cfg = _cfg(name, lens, H_q, H_kv, d_h, d_idx, k, prefix)
    if full:
        rows = np.arange(cfg.T)
    else:
        rng = np.random.default_rng(3)
        cu = cfg.cu_seqlens()
        fixed = [int(cu[s]) + r for s in range(len(lens)) for r in (0, 127, 128, lens[s] - 1) if r < lens[s]]
        rows = np.unique(np.concatenate([np.array(fixed), rng.choice(cfg.T, 400, replace=False)]))
    _check(cfg, rows)


def test_varlen_chunk_continuation_equals_full_prefill():
    """A 4000-token sequence processed as one prefill, and as a chunk of its last 1952 rows on top of
    a cached 2048-token prefix: identical selections and outputs on those rows."""
    full_cfg = _cfg("cont", (4000,), 16, 2, 128, 64, 6)
    inp, out_f, lse_f, bi_f = _run(full_cfg)
    pre = 2048
    t = {n: dev(inp[n]) for n in ("k", "v", "k_idx")}
    q = dev(np.ascontiguousarray(inp["q"][pre:]))
    q_idx = dev(np.ascontiguousarray(inp["q_idx"][pre:]))
    out_c, lse_c, bi_c = msa.msa_sparse_prefill_varlen(q, t["k"], t["v"], q_idx, t["k_idx"], [0, 4000 - pre], 128, 6,
                                                       cu_seqlens_k=[0, 4000])
    torch.cuda.synchronize()
    assert torch.equal(bi_c, bi_f[:, pre:, :])
    assert torch.equal(out_c, out_f[pre:])
    assert torch.equal(lse_c, lse_f[pre:])
