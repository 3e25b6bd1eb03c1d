"""Failure detection on the GPU without a fault: a bounded wait that can never complete expires,
the kernel records MSA_ERR_TIMEOUT in the device error word and returns, and the CUDA context
stays usable for normal work afterwards."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import block_sparse_long_idx_b200 as msa_pkg  # noqa: E402
import oracle  # noqa: E402
from block_sparse_long_idx_b200 import synth  # noqa: E402
from tests.gpu_util import (assert_lse_close, assert_out_close, assert_selection_equal, bf16_to_f64,  # noqa: E402
                            dev)

TIMEOUT = 5


@pytest.fixture(scope="module")
def msa():
    return msa_pkg


def test_bounded_wait_expires_and_reports_timeout(msa):
    ws = torch.zeros(msa.api.lib.msa_selftest_workspace_size(), dtype=torch.uint8, device="cuda")
    st = msa.msa_selftest_wait_timeout(limit_cycles=200_000, workspace=ws)  # ~0.1 ms of SM clock
    assert st == TIMEOUT, msa.status_string(st)
    word = ws[:8].view(torch.int32).cpu().tolist()
    assert word == [TIMEOUT, 900]  # status, waiting site of the self-test kernel


def test_context_usable_after_timeout(msa):
    assert msa.msa_selftest_wait_timeout(limit_cycles=50_000) == TIMEOUT
    cfg = synth.TINY
    inp = synth.prefill_inputs(cfg)
    t = {n: dev(a) for n, a in inp.items()}
    bi = msa.msa_index_topk(t["q_idx"], t["k_idx"], cfg.B_k, cfg.k)
    kv = msa.msa_build_kv2q(bi, cfg.B_k)
    out, lse = msa.msa_sparse_prefill(t["q"], t["k"], t["v"], bi, kv)
    torch.cuda.synchronize()
    rows = np.array([0, 1, cfg.B_k - 1, cfg.B_k, cfg.N // 2, cfg.N - 1])
    sel, want, want_lse = oracle.prefill_rows(inp, rows, cfg.B_k, cfg.k)
    assert_selection_equal(bi.cpu().numpy()[:, rows, :], np.ascontiguousarray(sel.transpose(1, 0, 2)), rows)
    assert_out_close(bf16_to_f64(out)[rows], want)
    assert_lse_close(lse.cpu().numpy()[rows].astype(np.float64), want_lse)
