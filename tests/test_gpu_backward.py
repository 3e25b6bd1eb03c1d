"""GPU parity, backward: dq, dk, dv of the CUDA path against the CPU oracle's gradients
(selections held fixed), on small shapes in full and on sampled rows / blocks, plus the two sums
that hold at any size (sum_j dv[j, r] = sum of the group's dout; sum_j dk[j, r] = 0) on the 128K
planted workload; and the index-branch KL alignment fused into the same pass (per-row KL, dq_idx,
dk_idx against the oracle; sum_j dk_idx[j, r] = 0 at 128K).

Tolerance (gradients are bf16 outputs of products whose operands P and dS are rounded to bf16,
accumulated in fp32; each rounding is 2^-9 relative): per tensor, max |d| <= 2e-2 * max |ref| + 1e-5
and mean |d| <= 1e-2 * mean |ref| + 1e-5. The absolute 1e-5 only matters where the reference vanishes
(a row whose token set is one token has a zero softmax Jacobian, so its dq is exactly 0, and the
kernel's dP - D then cancels to the rounding of the forward's bf16 output, ~1e-7).
"""
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
from tests.gpu_util import bf16_to_f64, dev  # noqa: E402

GRAD_MAX_REL = 2e-2
GRAD_MEAN_REL = 1e-2
GRAD_ATOL = 1e-5


def assert_grad_close(got, want, what):
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    d = np.abs(got - want)
    scale_max, scale_mean = float(np.abs(want).max()), float(np.abs(want).mean())
    mx, mean = float(d.max()), float(d.mean())
    assert mx <= GRAD_MAX_REL * scale_max + GRAD_ATOL and mean <= GRAD_MEAN_REL * scale_mean + GRAD_ATOL, (
        f"{what}: max |d| {mx:.3e} (ref max {scale_max:.3e}), mean |d| {mean:.3e} (ref mean {scale_mean:.3e}); "
        f"worst index {np.unravel_index(int(d.argmax()), d.shape)}")


def _cfg(name, N, H_q, H_kv, d_h, d_idx, k):
    return synth.PrefillConfig(name, N=N, H_q=H_q, H_kv=H_kv, d_h=d_h, d_idx=d_idx, B_k=128, k=k,
                               seed=zlib.crc32(name.encode()) % 1000)


def _forward_backward(cfg, inp, dout, use_kv=True, workspace=None):
    t = {n: dev(a) for n, a in inp.items()}
    bi = msa.msa_index_topk(t["q_idx"], t["k_idx"], 128, cfg.k)
    kv = msa.msa_build_kv2q(bi, 128)
    out, lse = msa.msa_sparse_prefill(t["q"], t["k"], t["v"], bi, kv)
    dq, dk, dv = msa.msa_sparse_backward(t["q"], t["k"], t["v"], out, lse, dev(dout), bi, kv if use_kv else None,
                                         workspace=workspace)
    torch.cuda.synchronize()
    return bf16_to_f64(dq), bf16_to_f64(dk), bf16_to_f64(dv)


CASES = [
    # name, N, H_q, H_kv, d_h, d_idx, k, full (all rows and blocks) or sampled
    ("tiny_N2048_G4", 2048, 8, 2, 64, 32, 4, True),
    ("ragged_G1_N1000", 1000, 2, 2, 128, 32, 3, True),
    ("k_over_blocks_G8_N777", 777, 16, 2, 64, 64, 16, True),
    ("one_row", 1, 4, 1, 128, 64, 3, True),
    ("G16_dh128_N1500", 1500, 32, 2, 128, 64, 8, False),
    ("G2_N3000_k1", 3000, 4, 2, 128, 64, 1, False),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_backward_small(case):
    name, N, H_q, H_kv, d_h, d_idx, k, full = case
    cfg = _cfg(name, N, H_q, H_kv, d_h, d_idx, k)
    inp = synth.prefill_inputs(cfg)
    dout = synth.normal_bf16((N, H_q, d_h), cfg.seed, "dout")
    dq, dk, dv = _forward_backward(cfg, inp, dout)
    sel = oracle.select_rows(inp["q_idx"], inp["k_idx"], np.arange(N), 128, k)  # [N, H_kv, k]
    nb = (N + 127) // 128
    rows = np.arange(N) if full else synth.sample_rows(N, 128, 200, 3)
    want_dq = oracle.backward_dq_rows(inp["q"], dout, inp["k"], inp["v"], rows, sel[rows], 128)
    assert_grad_close(dq[rows], want_dq, "dq")
    if full:
        pairs = [(r, b) for r in range(H_kv) for b in range(nb)]
    else:
        pairs = sorted({(0, 0), (H_kv - 1, nb - 1), (0, nb // 2), (H_kv - 1, 1)})
    want_dk, want_dv = oracle.backward_dkv_blocks(inp["q"], dout, inp["k"], inp["v"], sel, pairs, 128)
    for x, (r, b) in enumerate(pairs):
        lo, hi = b * 128, min(N, (b + 1) * 128)
        want_dk[x, hi - lo:] = 0.0
    got_dk = np.stack([np.pad(dk[b * 128:(b + 1) * 128, r], ((0, 128 - len(dk[b * 128:(b + 1) * 128])), (0, 0)))
                       for r, b in pairs])
    got_dv = np.stack([np.pad(dv[b * 128:(b + 1) * 128, r], ((0, 128 - len(dv[b * 128:(b + 1) * 128])), (0, 0)))
                       for r, b in pairs])
    assert_grad_close(got_dk, want_dk, "dk")
    assert_grad_close(got_dv, want_dv, "dv")


def test_backward_internal_inversion_and_error_word():
    """Without a built inversion the call builds one in its workspace; the device error word stays clear."""
    cfg = _cfg("internal", 1300, 8, 2, 64, 32, 5)
    inp = synth.prefill_inputs(cfg)
    dout = synth.normal_bf16((cfg.N, cfg.H_q, cfg.d_h), cfg.seed, "dout")
    nbytes = msa.lib.msa_sparse_backward_workspace_size(cfg.N, cfg.H_q, cfg.H_kv, cfg.d_h, 128, cfg.k, 0, 1)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    dq, dk, dv = _forward_backward(cfg, inp, dout, use_kv=False, workspace=ws)
    assert msa.msa_get_device_error(ws) == 0
    sel = oracle.select_rows(inp["q_idx"], inp["k_idx"], np.arange(cfg.N), 128, cfg.k)
    want_dq = oracle.backward_dq_rows(inp["q"], dout, inp["k"], inp["v"], np.arange(cfg.N), sel, 128)
    assert_grad_close(dq, want_dq, "dq")
    nb = (cfg.N + 127) // 128
    pairs = [(r, b) for r in range(cfg.H_kv) for b in range(nb)]
    want_dk, want_dv = oracle.backward_dkv_blocks(inp["q"], dout, inp["k"], inp["v"], sel, pairs, 128)
    tok = lambda g: g.reshape(cfg.H_kv, nb * 128, -1)[:, :cfg.N].transpose(1, 0, 2)  # noqa: E731
    assert_grad_close(dk, tok(want_dk), "dk")
    assert_grad_close(dv, tok(want_dv), "dv")


def test_backward_128k_planted_sampled():
    """The 128K planted workload: dq on sampled rows against the oracle (its own selections of those
    rows), and the two column sums of dk and dv that hold at any size."""
    cfg = synth.P128K
    inp = synth.prefill_inputs(cfg)
    dout = synth.normal_bf16((cfg.N, cfg.H_q, cfg.d_h), cfg.seed, "dout")
    dq, dk, dv = _forward_backward(cfg, inp, dout)
    rows = synth.sample_rows(cfg.N, 128, 48, 11)
    sel = oracle.select_rows(inp["q_idx"], inp["k_idx"], rows, 128, cfg.k)
    want_dq = oracle.backward_dq_rows(inp["q"], dout, inp["k"], inp["v"], rows, sel, 128)
    assert_grad_close(dq[rows], want_dq, "dq (sampled rows)")
    G = cfg.H_q // cfg.H_kv
    dO = bf16_to_f64(torch.from_numpy(dout.view(np.int16)))
    for r in range(cfg.H_kv):
        want = dO[:, r * G:(r + 1) * G].sum(axis=(0, 1))        # attention weights of a row sum to one
        got = dv[:, r].sum(axis=0)
        assert np.max(np.abs(got - want)) <= 1e-2 * np.abs(dv[:, r]).sum(axis=0).max(), r
        sk = dk[:, r].sum(axis=0)                                # softmax Jacobian rows sum to zero
        assert np.max(np.abs(sk)) <= 1e-2 * np.abs(dk[:, r]).sum(axis=0).max(), r


def _forward_backward_kl(cfg, inp, dout, w):
    t = {n: dev(a) for n, a in inp.items()}
    bi = msa.msa_index_topk(t["q_idx"], t["k_idx"], 128, cfg.k)
    kv = msa.msa_build_kv2q(bi, 128)
    out, lse = msa.msa_sparse_prefill(t["q"], t["k"], t["v"], bi, kv)
    res = msa.msa_sparse_backward(t["q"], t["k"], t["v"], out, lse, dev(dout), bi, kv, q_idx=t["q_idx"],
                                  k_idx=t["k_idx"], kl_weight=w)
    torch.cuda.synchronize()
    dq, dk, dv, dqi, dki, kl = res
    return (bf16_to_f64(dq), bf16_to_f64(dk), bf16_to_f64(dv), bf16_to_f64(dqi), bf16_to_f64(dki),
            kl.cpu().numpy().astype(np.float64))


KL_CASES = [
    # name, N, H_q, H_kv, d_h, d_idx, k, full
    ("kl_tiny_N2048_G4_didx32", 2048, 8, 2, 64, 32, 4, True),
    ("kl_G16_N1500_didx64", 1500, 32, 2, 128, 64, 8, False),
    ("kl_G1_N700", 700, 2, 2, 128, 64, 3, True),
]


@pytest.mark.parametrize("case", KL_CASES, ids=[c[0] for c in KL_CASES])
def test_backward_with_kl(case):
    """The KL alignment's per-(row, group) value and gradients in q_idx and k_idx, and the main-branch
    gradients of the same call (the KL part must leave them as without it)."""
    name, N, H_q, H_kv, d_h, d_idx, k, full = case
    cfg = _cfg(name, N, H_q, H_kv, d_h, d_idx, k)
    inp = synth.prefill_inputs(cfg)
    dout = synth.normal_bf16((N, H_q, d_h), cfg.seed, "dout")
    w = 0.5
    dq, dk, dv, dqi, dki, kl = _forward_backward_kl(cfg, inp, dout, w)
    sel = oracle.select_rows(inp["q_idx"], inp["k_idx"], np.arange(N), 128, k)
    rows = np.arange(N) if full else synth.sample_rows(N, 128, 200, 5)
    want_kl, want_dqi = oracle.kl_rows(inp["q"], inp["q_idx"], inp["k"], inp["k_idx"], rows, sel[rows], 128, w)
    assert_grad_close(kl[rows], want_kl, "kl")
    assert_grad_close(dqi[rows], want_dqi, "dq_idx")
    want_dq = oracle.backward_dq_rows(inp["q"], dout, inp["k"], inp["v"], rows, sel[rows], 128)
    assert_grad_close(dq[rows], want_dq, "dq")
    nb = (N + 127) // 128
    pairs = ([(r, b) for r in range(H_kv) for b in range(nb)] if full
             else sorted({(0, 0), (H_kv - 1, nb - 1), (0, nb // 2), (H_kv - 1, 1)}))
    want_dki = oracle.kl_dk_idx_blocks(inp["q"], inp["q_idx"], inp["k"], inp["k_idx"], sel, pairs, 128, w)
    got_dki = np.stack([np.pad(dki[b * 128:(b + 1) * 128, r], ((0, 128 - len(dki[b * 128:(b + 1) * 128])), (0, 0)))
                        for r, b in pairs])
    assert_grad_close(got_dki, want_dki, "dk_idx")
    want_dk, want_dv = oracle.backward_dkv_blocks(inp["q"], dout, inp["k"], inp["v"], sel, pairs, 128)
    got_dv = np.stack([np.pad(dv[b * 128:(b + 1) * 128, r], ((0, 128 - len(dv[b * 128:(b + 1) * 128])), (0, 0)))
                       for r, b in pairs])
    assert_grad_close(got_dv, want_dv, "dv")


def test_backward_kl_128k_planted_sampled():
    """The 128K planted workload with the KL part: KL and dq_idx on sampled rows against the oracle
    (its own selections of those rows), and sum_j dk_idx[j, r] = 0 (student and teacher both sum to
    one over every row's token set)."""
    cfg = synth.P128K
    inp = synth.prefill_inputs(cfg)
    dout = synth.normal_bf16((cfg.N, cfg.H_q, cfg.d_h), cfg.seed, "dout")
    w = 1.0 / (cfg.N * cfg.H_kv)
    _, _, _, dqi, dki, kl = _forward_backward_kl(cfg, inp, dout, w)
    rows = synth.sample_rows(cfg.N, 128, 48, 13)
    sel = oracle.select_rows(inp["q_idx"], inp["k_idx"], rows, 128, cfg.k)
    want_kl, want_dqi = oracle.kl_rows(inp["q"], inp["q_idx"], inp["k"], inp["k_idx"], rows, sel, 128, w)
    assert_grad_close(kl[rows], want_kl, "kl (sampled rows)")
    assert_grad_close(dqi[rows] / w, want_dqi / w, "dq_idx (sampled rows)")
    for r in range(cfg.H_kv):
        s = dki[:, r].sum(axis=0)
        assert np.max(np.abs(s)) <= 1e-2 * np.abs(dki[:, r]).sum(axis=0).max(), r

