"""GPU parity, prefill path, small shapes: selections (bit-exact), KV->Q inversion (exact) and attention
outputs (tolerance) against the CPU oracle. Shapes span several tiles, ragged tails, k larger than the
visible block count, G from 1 to 64, d_h 64/128, d_idx 32/64/128, and multi-pass prefill."""
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
from tests.gpu_util import (assert_lse_close, assert_out_close, assert_selection_equal, bf16_to_f64, check_kv2q,  # noqa: E402
                            dev)

CASES = [
    # name, N, H_q, H_kv, d_h, d_idx, k, full_rows
    ("tiny_N2048_G4", 2048, 8, 2, 64, 32, 4, True),
    ("ragged_N1000", 1000, 8, 2, 64, 32, 4, True),
    ("single_tile_N100", 100, 4, 1, 64, 64, 2, True),
    ("one_row", 1, 4, 1, 64, 64, 3, True),
    ("G16_dh128_N4173", 4173, 32, 2, 128, 64, 16, False),
    ("k1_N700", 700, 8, 2, 128, 64, 1, True),
    ("didx128_G8_N1500", 1500, 16, 2, 128, 128, 8, False),
    ("G1_N600", 600, 2, 2, 64, 64, 5, True),
    ("G64_N400", 400, 64, 1, 128, 64, 3, False),
]


def _cfg(name, N, H_q, H_kv, d_h, d_idx, k):
    return synth.PrefillConfig(name, N=N, H_q=H_q, H_kv=H_kv, d_h=d_h, d_idx=d_idx, B_k=128, k=k,
                               seed=zlib.crc32(name.encode()) % 1000)


def _run(cfg, rows, window=0, chunk=0, max_rows_per_pass=0, inputs=None):
    inp = inputs if inputs is not None else synth.prefill_inputs(cfg)
    t = {n: dev(a) for n, a in inp.items()}
    bi = msa.msa_index_topk(t["q_idx"], t["k_idx"], 128, cfg.k)
    kv = msa.msa_build_kv2q(bi, 128, window, chunk)
    out, lse = msa.msa_sparse_prefill(t["q"], t["k"], t["v"], bi, kv, max_rows_per_pass=max_rows_per_pass)
    torch.cuda.synchronize()
    sel_all = oracle.select_all(inp["q_idx"], inp["k_idx"], 128, cfg.k)
    assert_selection_equal(bi.cpu().numpy(), sel_all)
    check_kv2q(kv, sel_all, oracle)
    sel_rows = np.ascontiguousarray(sel_all[:, rows, :].transpose(1, 0, 2))
    want, want_lse = oracle.attend_rows(inp["q"], inp["k"], inp["v"], rows, sel_rows, 128)
    got = bf16_to_f64(out)[rows]
    assert_out_close(got, want)
    assert_lse_close(lse.cpu().numpy()[rows].astype(np.float64), want_lse)


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_prefill_small(case):
    name, N, H_q, H_kv, d_h, d_idx, k, full = case
    cfg = _cfg(name, N, H_q, H_kv, d_h, d_idx, k)
    rows = np.arange(N) if full else synth.sample_rows(N, 128, 384, 7)
    _run(cfg, rows)


def test_prefill_small_windows_and_passes():
    """Small query windows / chunks and a workspace that forces several passes."""
    cfg = _cfg("passes", 3000, 8, 2, 64, 32, 4)
    _run(cfg, np.arange(3000), window=256, chunk=16, max_rows_per_pass=512)


def test_prefill_all_ties():
    """q_idx == 0: every pooled score ties, the lowest blocks win (closed form checked by the oracle pins)."""
    cfg = _cfg("ties", 1500, 8, 2, 64, 64, 6)
    inp = synth.prefill_inputs(cfg)
    inp["q_idx"] = np.zeros_like(inp["q_idx"])
    _run(cfg, np.arange(1500), inputs=inp)


def test_prefill_planted_hot_blocks():
    """Planted recipe on a small sequence: hot blocks selected by many rows (load-balance path)."""
    cfg = synth.PrefillConfig("planted_small", N=8192, H_q=32, H_kv=2, d_h=128, d_idx=64, B_k=128, k=16, seed=9,
                              planted=True, n_needles=8)
    _run(cfg, synth.sample_rows(8192, 128, 256, 3))
