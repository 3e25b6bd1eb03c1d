"""GPU parity, decode path, small shapes: selections (bit-exact) and outputs (tolerance) vs the oracle,
including lengths 1, one block, one block + 1 and L_max, and a rejected out-of-range length."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import block_sparse_long_idx_b200 as msa  # noqa: E402
import oracle  # noqa: E402
from block_sparse_long_idx_b200 import synth  # noqa: E402
from tests.gpu_util import assert_lse_close, assert_out_close, bf16_to_f64, dev  # noqa: E402


def _decode_case(B, L_max, H_q, H_kv, d_h, d_idx, k, lens, seed):
    cfg = synth.DecodeConfig("dec", B=B, L_max=L_max, len_lo=1, len_hi=L_max, H_q=H_q, H_kv=H_kv, d_h=d_h,
                             d_idx=d_idx, B_k=128, k=k, seed=seed)
    inp = synth.decode_inputs(cfg, lens=np.asarray(lens, dtype=np.int32))
    t = {n: dev(a) for n, a in inp.items()}
    out, lse, bi = msa.msa_sparse_decode(t["q"], t["q_idx"], t["k_cache"], t["v_cache"], t["k_idx_cache"], t["lens"],
                                         128, k)
    torch.cuda.synchronize()
    sel, want, want_lse = oracle.decode(inp, 128, k)
    assert np.array_equal(bi.cpu().numpy(), sel), "decode selection differs"
    assert_out_close(bf16_to_f64(out), want)
    assert_lse_close(lse.cpu().numpy().astype(np.float64), want_lse)


@pytest.mark.parametrize("shape", [(8, 2000, 32, 2, 128, 64, 16), (6, 1100, 8, 2, 64, 32, 4),
                                   (5, 3000, 16, 4, 128, 32, 8)], ids=["G16", "G4_small", "G4_didx32"])
def test_decode_small(shape):
    B, L_max, H_q, H_kv, d_h, d_idx, k = shape
    rng = np.random.default_rng(B)
    lens = [1, 128, 129, L_max] + list(rng.integers(1, L_max + 1, size=B - 4))
    _decode_case(B, L_max, H_q, H_kv, d_h, d_idx, k, lens[:B], seed=B)


def test_decode_rejects_bad_length():
    """A length outside [1, L_max] sets MSA_ERR_DEVICE_CHECK; the other sequences are still correct."""
    B, L_max, H_q, H_kv, d_h, d_idx, k = 3, 600, 8, 2, 64, 32, 4
    cfg = synth.DecodeConfig("bad", B=B, L_max=L_max, len_lo=1, len_hi=L_max, H_q=H_q, H_kv=H_kv, d_h=d_h,
                             d_idx=d_idx, B_k=128, k=k, seed=3)
    inp = synth.decode_inputs(cfg, lens=np.array([300, L_max + 5, 600], dtype=np.int32))
    t = {n: dev(a) for n, a in inp.items()}
    ws = torch.empty(msa.api.lib.msa_sparse_decode_workspace_size(B, L_max, H_q, H_kv, d_h, d_idx, 128, k),
                     dtype=torch.uint8, device="cuda")
    out, lse, bi = msa.msa_sparse_decode(t["q"], t["q_idx"], t["k_cache"], t["v_cache"], t["k_idx_cache"], t["lens"],
                                         128, k, workspace=ws)
    assert msa.msa_get_device_error(ws) == 6
    ok = {n: (a[[0, 2]] if n != "lens" else a[[0, 2]]) for n, a in inp.items()}
    sel, want, want_lse = oracle.decode(ok, 128, k)
    got = bf16_to_f64(out)[[0, 2]]
    assert_out_close(got, want)
    assert (bi.cpu().numpy()[1] == -1).all()


def test_decode_cuda_graph_replay():
    """The decode step (pooling, Top-k, split attention, combine and their memsets) captured once in a
    CUDA graph and replayed gives the eager result bit for bit; new cache contents and lengths
    written into the same buffers between replays are picked up."""
    cfg = synth.DecodeConfig("graph", B=6, L_max=1500, len_lo=1, len_hi=1500, H_q=32, H_kv=2, d_h=128, d_idx=64,
                             B_k=128, k=8, seed=41)
    inp = synth.decode_inputs(cfg, lens=np.array([1, 128, 700, 1500, 129, 1000], dtype=np.int32))
    t = {n: dev(a) for n, a in inp.items()}
    out = torch.empty_like(t["q"])
    lse = torch.empty((cfg.B, cfg.H_q), dtype=torch.float32, device="cuda")
    bi = torch.empty((cfg.B, cfg.H_kv, cfg.k), dtype=torch.int32, device="cuda")
    ws = torch.empty(msa.api.lib.msa_sparse_decode_workspace_size(cfg.B, cfg.L_max, cfg.H_q, cfg.H_kv, cfg.d_h,
                                                                  cfg.d_idx, 128, cfg.k), dtype=torch.uint8,
                     device="cuda")

    def step():
        msa.msa_sparse_decode(t["q"], t["q_idx"], t["k_cache"], t["v_cache"], t["k_idx_cache"], t["lens"], 128, cfg.k,
                              out=out, lse=lse, block_idx_out=bi, workspace=ws)

    step()
    torch.cuda.synchronize()
    eager = (out.clone(), lse.clone(), bi.clone())
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()  # warm the launch path on the capture stream
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager[0]) and torch.equal(lse, eager[1]) and torch.equal(bi, eager[2])
    # the next token of every sequence: new inputs in the same buffers, one more replay
    inp2 = synth.decode_inputs(cfg.with_(seed=42), lens=np.array([2, 129, 701, 1500, 130, 1001], dtype=np.int32))
    for n, a in inp2.items():
        t[n].copy_(dev(a))
    g.replay()
    torch.cuda.synchronize()
    sel, want, want_lse = oracle.decode(inp2, 128, cfg.k)
    assert np.array_equal(bi.cpu().numpy(), sel)
    assert_out_close(bf16_to_f64(out), want)
    assert_lse_close(lse.cpu().numpy().astype(np.float64), want_lse)
