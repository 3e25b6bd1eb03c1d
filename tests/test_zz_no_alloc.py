"""msa_build_kv2q_static, the KV->Q inversion for callers that cannot allocate device memory.

Such callers (a plug-in handed only its input and output buffers by a host framework that owns all
device memory, or a latency-critical loop where cudaMalloc/cudaFree would synchronise the device)
cannot provide a workspace; this entry point keeps its scratch in a fixed 1 MiB array of the
library instead. The test calls it through the C ABI twice in a row, on two different inputs, and
checks each result against the workspace entry point msa_build_kv2q, bit for bit (integer work).
It lives in a file of its own that pytest collects last.
"""
import ctypes

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import block_sparse_long_idx_b200 as msa  # noqa: E402
from block_sparse_long_idx_b200 import synth  # noqa: E402
from tests.gpu_util import dev  # noqa: E402


def _selection(seed):
    cfg = synth.PrefillConfig("no_alloc", N=5000, H_q=32, H_kv=2, d_h=128, d_idx=64, B_k=128, k=16, seed=seed)
    inp = synth.prefill_index_inputs(cfg)
    return msa.msa_index_topk(dev(inp["q_idx"]), dev(inp["k_idx"]), 128, cfg.k)


def _arrays(kv: "msa.KV2Q"):
    n = int(kv.window_items().cpu().numpy()[-1])
    return {"offsets": kv.offsets().cpu().numpy(), "entries": kv.entries().cpu().numpy(),
            "window_items": kv.window_items().cpu().numpy(), "items": kv.items(n).cpu().numpy()}


def test_static_scratch_matches_workspace_entry_point():
    stream = torch.cuda.current_stream().cuda_stream
    for seed in (11, 12):  # two calls in a row on different inputs: no state may leak between them
        bi = _selection(seed)
        H_kv, N, k = bi.shape
        want = _arrays(msa.msa_build_kv2q(bi, 128))
        L = msa.msa_kv2q_layout_get(N, H_kv, 128, k)
        buf = torch.full((L.total_bytes,), 0x5A, dtype=torch.uint8, device="cuda")
        st = msa.lib.msa_build_kv2q_static(bi.data_ptr(), ctypes.byref(L), buf.data_ptr(), stream)
        assert st == 0, msa.status_string(st)
        torch.cuda.synchronize()
        got = _arrays(msa.KV2Q(L, buf))
        for name in ("offsets", "window_items", "items"):
            assert np.array_equal(got[name], want[name]), name
        for r in range(H_kv):
            n = int(want["offsets"][r, -1])
            assert np.array_equal(got["entries"][r, :n], want["entries"][r, :n]), f"entries of group {r}"


def test_static_scratch_rejects_bad_layout():
    bi = _selection(13)
    H_kv, N, k = bi.shape
    L = msa.msa_kv2q_layout_get(N, H_kv, 128, k)
    L.total_bytes += 256  # not a layout the library produced
    buf = torch.empty(L.total_bytes, dtype=torch.uint8, device="cuda")
    st = msa.lib.msa_build_kv2q_static(bi.data_ptr(), ctypes.byref(L), buf.data_ptr(),
                                       torch.cuda.current_stream().cuda_stream)
    assert st == 1  # MSA_ERR_INVALID_ARG


def test_static_scratch_rejects_edited_block_count():
    """A layout whose nb or n_windows was edited would size the kernels' counters past the kv2q
    buffer; the entry point rejects it before enqueueing anything."""
    bi = _selection(14)
    H_kv, N, k = bi.shape
    buf = torch.empty(msa.msa_kv2q_layout_get(N, H_kv, 128, k).total_bytes, dtype=torch.uint8, device="cuda")
    for field in ("nb", "n_windows"):
        L = msa.msa_kv2q_layout_get(N, H_kv, 128, k)
        setattr(L, field, getattr(L, field) + 1)
        st = msa.lib.msa_build_kv2q_static(bi.data_ptr(), ctypes.byref(L), buf.data_ptr(),
                                           torch.cuda.current_stream().cuda_stream)
        assert st == 1, field  # MSA_ERR_INVALID_ARG
