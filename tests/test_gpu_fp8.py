"""FP8 main branch ("MiniMax M3" blog post, kernel paragraph: FP8 tensor cores) on the GPU against the
oracle's reading: per-(token, head) E4M3 quantisation (scale = amax / 448, nearest code, ties to the
even code, saturating) and exact attention over the dequantised values.

Quantisation is compared bit for bit: codes, the fp32 rounding of the oracle's fp64 scales, their
reciprocals and the per-block scale maxima.

Tolerance of the FP8 attention (derived from what the kernel rounds). The S and PV products
accumulate in fp32 (relative error ~1e-7 on these sizes); the one coarse rounding is the attention
weight P' = P * s_v * C_b rounded to E4M3 for the PV product: a relative error delta_j with
|delta_j| <= 2^-4 (3 mantissa bits; subnormal codes lie below 2^-6 of the block's largest weight, an
absolute error under 2^-10 / 448 relative to it). Each partial output is normalised by the sum of the
weights those codes stand for, so it stays an exact weighted average of V rows and, to first order,
out - exact = sum_j w_j delta_j (v_j - out) over the row's tokens T. With delta_j independent and
uniform (sigma = 2^-4 / sqrt(3)), v ~ N(0, 1) and logits of unit spread (||w||_2 ~ e^(1/2) / sqrt(|T|)):
sigma(|T|) = 2^-4 / sqrt(3) * e^(1/2) / sqrt(|T|). The bf16 output adds at most 2^-9 |out| <= 2^-7
for |out| <= 4. The test allows, per row, max |d| <= 6 sigma(|T|) + 2^-7 (a one-token row is exact:
its only weight normalises to 1), and over all values mean |d| <= 1.5 * mean_i(0.8 sigma(|T_i|)) +
2^-10 (0.8 sigma is the mean of |N(0, sigma)|; 2^-10 covers the mean bf16 rounding)."""
import math

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import block_sparse_long_idx_b200 as msa  # noqa: E402
import oracle  # noqa: E402
from block_sparse_long_idx_b200 import synth  # noqa: E402
from tests.gpu_util import assert_selection_equal, bf16_to_f64, dev  # noqa: E402

SIGMA1 = 2.0 ** -4 / math.sqrt(3.0) * math.exp(0.5)  # sigma(|T|) * sqrt(|T|)


def _oracle_quant(x):
    """Oracle codes [N, H, d] and fp64 scales [N, H]."""
    return oracle.default().quantize_e4m3(x)


def _check_quant(x, q, rows=None):
    """GPU codes and scales of x against the oracle's, on every row or on the given token rows (the
    oracle then quantises only those: codes [n, H, d], scales [n, H])."""
    N, H, d = x.shape
    sub = rows is not None
    codes, scales = _oracle_quant(x[rows] if sub else x)
    got = q.codes.cpu().numpy()
    if sub:
        got = got[rows]
    if not np.array_equal(got, codes):
        bad = np.argwhere(got != codes)[0]
        raise AssertionError(f"code differs at {tuple(bad)}: got {got[tuple(bad)]:#04x} want {codes[tuple(bad)]:#04x}")
    S = q.scales.shape[1]
    gs = q.scales.cpu().numpy()
    assert np.array_equal(gs[:, rows] if sub else gs[:, :N], scales.T.astype(np.float32)), "scales"
    assert (gs[:, N:] == 1.0).all(), "padding scales"
    gr = q.rscales.cpu().numpy()
    assert np.array_equal(gr[:, rows] if sub else gr[:, :N], (1.0 / scales.T).astype(np.float32)), "reciprocals"
    if not sub:
        want_max = np.zeros((H, S // 128), dtype=np.float32)
        s32 = scales.T.astype(np.float32)
        for b in range(S // 128):
            want_max[:, b] = s32[:, b * 128:(b + 1) * 128].max(axis=1)
        assert np.array_equal(q.blkmax.cpu().numpy(), want_max), "block maxima"
    return codes, scales


def test_quantize_e4m3_bit_exact():
    """Random rows plus rows that hit the definition's edge cases."""
    rng = np.random.default_rng(7)
    N, H, d = 300, 4, 128
    x = synth.normal_bf16((N, H, d), 3, "fp8q")
    x = x.copy()
    x[5, 1, :] = 0                                       # all-zero row: scale 1, codes 0
    x[6, 2, :] = 0x8000                                  # negative zeros: code 0x80
    # amax = 3.5 -> scale = 2^-7 exactly: quotients x * 128 land on code midpoints (ties to even)
    mids = np.array([1.0625, 1.1875, 2.125, 0.0146484375, 0.01171875, 432.0 / 128, -1.0625, -2.375],
                    dtype=np.float32)
    row = np.zeros(d, dtype=np.float32)
    row[0] = 3.5
    row[1:1 + len(mids)] = mids
    row[20:30] = np.array([2 ** -12, 2 ** -14, 2 ** -15, 3 * 2 ** -16, 7.5 * 2 ** -16, -2 ** -13, 1e-30, 3.4,
                           3.49, -3.5], dtype=np.float32)
    x[7, 0, :] = synth.f32_to_bf16_bits(row)
    x[8, 3, :] = synth.f32_to_bf16_bits(rng.standard_normal(d).astype(np.float32) * 1e-3)  # small amax
    # amax below 448 * FLT_MIN: 448 / amax overflows fp32, the definition's fp64 quotient does not
    x[9, 0, :] = synth.f32_to_bf16_bits(rng.standard_normal(d).astype(np.float32) * np.float32(1e-37))
    xd = dev(x)
    q = msa.msa_quantize_e4m3(xd)
    torch.cuda.synchronize()
    codes, _ = _check_quant(x, q)
    assert codes[5, 1].max() == 0 and (codes[6, 2] == 0x80).all()


def _visible_counts(sel, rows, B_k):
    """|T(i)| per requested row: visible tokens of the selected blocks."""
    T = np.zeros(len(rows), dtype=np.int64)
    for t, i in enumerate(rows):
        for b in sel[t, 0]:
            if b >= 0:
                T[t] += min(B_k, int(i) - int(b) * B_k + 1)
    return T


def run_fp8(cfg, n_rows=0):
    inp = synth.prefill_inputs(cfg)
    t = {n: dev(a) for n, a in inp.items()}
    qq, kq, vq = (msa.msa_quantize_e4m3(t[n]) for n in ("q", "k", "v"))
    bi = msa.msa_index_topk(t["q_idx"], t["k_idx"], cfg.B_k, cfg.k)
    kv = msa.msa_build_kv2q(bi, cfg.B_k)
    ws = torch.empty(msa.msa_sparse_prefill_workspace_size(cfg.N, cfg.H_q, cfg.H_kv, cfg.d_h, cfg.B_k, cfg.k),
                     dtype=torch.uint8, device="cuda")
    out, lse = msa.msa_sparse_prefill_fp8(qq, kq, vq, bi, kv, workspace=ws)
    torch.cuda.synchronize()
    assert msa.msa_get_device_error(ws) == 0
    rows = np.arange(cfg.N) if n_rows == 0 else synth.sample_rows(cfg.N, cfg.B_k, n_rows, cfg.seed)
    kc, ks = _check_quant(inp["k"], kq)
    vc, vs = _check_quant(inp["v"], vq)
    # q: every row, or only the sampled rows (the oracle's attention reads q at the requested rows)
    qc_r, qs_r = _check_quant(inp["q"], qq, None if n_rows == 0 else rows)
    qc = np.zeros((cfg.N,) + qc_r.shape[1:], dtype=np.uint8)
    qs = np.ones((cfg.N, qc_r.shape[1]), dtype=np.float64)
    qc[rows], qs[rows] = qc_r, qs_r
    o = oracle.default()
    sel = o.select_rows(inp["q_idx"], inp["k_idx"], rows, cfg.B_k, cfg.k)
    assert_selection_equal(np.ascontiguousarray(bi.cpu().numpy()[:, rows, :]), np.ascontiguousarray(sel.transpose(1, 0, 2)),
                           rows)
    want, want_lse = o.attend_rows_e4m3((qc, qs), (kc, ks), (vc, vs), rows, sel, cfg.B_k)
    got = bf16_to_f64(out[torch.from_numpy(rows).cuda()])
    d = np.abs(got - want)
    assert np.isfinite(got).all()
    T = _visible_counts(sel, rows, cfg.B_k)
    tol = 6.0 * SIGMA1 / np.sqrt(T) + 2.0 ** -7
    worst = (d.max(axis=(1, 2)) / tol)
    i = int(worst.argmax())
    assert worst.max() <= 1.0, (f"row {rows[i]} (|T| = {T[i]}): max |d| = {d[i].max():.3e} > {tol[i]:.3e}")
    mean_tol = 1.5 * float(np.mean(0.8 * SIGMA1 / np.sqrt(T))) + 2.0 ** -10
    assert d.mean() <= mean_tol, f"mean |d| = {d.mean():.3e} > {mean_tol:.3e}"
    dl = np.abs(lse[torch.from_numpy(rows).cuda()].cpu().numpy().astype(np.float64) - want_lse)
    assert dl.max() <= 1e-3, f"lse max |d| = {dl.max():.3e}"
    return float(d.max()), float(d.mean())


def test_fp8_prefill_g4_ragged():
    """G = 4 (per-chunk query gather), ragged N, every row."""
    run_fp8(synth.PrefillConfig("fp8_g4", N=1000, H_q=16, H_kv=4, d_h=128, d_idx=32, B_k=128, k=4, seed=21))


def test_fp8_prefill_g16_all_rows():
    """The paper's head shape (G = 16, one TMA box per position), k = 16, every row."""
    run_fp8(synth.PrefillConfig("fp8_g16", N=4096, H_q=64, H_kv=4, d_h=128, d_idx=64, B_k=128, k=16, seed=22))


def test_fp8_prefill_32k_sampled():
    """The 32K configuration on 1024 sampled rows (k and v quantisation checked on every row)."""
    run_fp8(synth.P32K, 1024)


def test_fp8_prefill_128k_planted_sampled():
    """The 128K planted sequence on 512 sampled rows."""
    run_fp8(synth.P128K, 512)
