"""The C ABI on the host, no GPU needed: the library loads, exports every symbol include/msa.h declares,
rejects bad arguments with the documented status before touching the device, sizes its workspaces,
and honours host-side fault injection."""
import ctypes
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "msa.h")

OK, INVALID, UNSUPPORTED, WORKSPACE, CUDA = 0, 1, 2, 3, 4
P, P2, WS = 0x100000, 0x200000, 0x300000  # fake, suitably aligned device addresses (never dereferenced)


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MSA_API\s+[\w\s\*]*?\b(msa_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def msa():
    from block_sparse_long_idx_b200 import build

    if not os.path.exists(build.LIB):
        build.build()
    import block_sparse_long_idx_b200 as m

    return m


def test_every_declared_symbol_is_exported(msa):
    names = declared_symbols()
    assert len(names) >= 15
    raw = ctypes.CDLL(msa.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), n
    bound = {s[0] for s in msa.SIGNATURES}
    assert set(names) <= bound, set(names) - bound


def test_status_strings(msa):
    assert msa.status_string(0) == "MSA_OK"
    assert msa.status_string(3) == "MSA_ERR_WORKSPACE"
    assert msa.status_string(6) == "MSA_ERR_DEVICE_CHECK"


def test_index_topk_validation(msa):
    f = msa.lib.msa_index_topk
    assert f(None, P2, 1024, 2, 64, 128, 4, P, WS, 256, None) == INVALID        # null input
    assert f(P + 2, P2, 1024, 2, 64, 128, 4, P, WS, 256, None) == INVALID       # misaligned
    assert f(P, P2, 0, 2, 64, 128, 4, P, WS, 256, None) == INVALID              # N < 1
    assert f(P, P2, 1024, 2, 48, 128, 4, P, WS, 256, None) == UNSUPPORTED       # d_idx
    assert f(P, P2, 1024, 2, 64, 64, 4, P, WS, 256, None) == UNSUPPORTED        # B_k != 128
    assert f(P, P2, 1024, 2, 64, 128, 17, P, WS, 256, None) == UNSUPPORTED      # k > 16
    assert f(P, P2, 1024, 2, 64, 128, 4, P, WS, 16, None) == WORKSPACE          # workspace too small


def test_layout_and_workspace_sizes(msa):
    L = msa.msa_kv2q_layout_get(131072, 4, 128, 16)
    assert L.nb == 1024 and L.n_windows == 64 and L.window == 2048 and L.chunk == 512
    assert L.entries > L.offsets and L.total_bytes > L.bases
    with pytest.raises(msa.MsaError):
        msa.msa_kv2q_layout_get(1000, 2, 128, 4, window=100)    # window not a multiple of B_k
    ws = msa.api.lib.msa_sparse_prefill_workspace_size(131072, 64, 4, 128, 128, 16, 0, 0)
    assert ws > 131072 * 16 * 64 * 260                           # holds every partial of one pass
    ws8 = msa.api.lib.msa_sparse_prefill_workspace_size(131072, 64, 4, 128, 128, 16, 8192, 0)
    assert ws8 < ws / 10                                         # a pass cap shrinks it
    assert msa.api.lib.msa_sparse_decode_workspace_size(64, 131072, 64, 4, 128, 64, 128, 16) > 0


def test_prefill_and_decode_validation(msa):
    L = msa.msa_kv2q_layout_get(1024, 2, 128, 4)
    pf = msa.lib.msa_sparse_prefill
    # H_q % H_kv != 0
    assert pf(P, P, P, 1024, 6, 4, 128, 128, 4, P, None, None, P, None, WS, 1 << 30, None) == INVALID
    # d_h unsupported
    assert pf(P, P, P, 1024, 8, 2, 96, 128, 4, P, None, None, P, None, WS, 1 << 30, None) == UNSUPPORTED
    # layout given without buffer
    assert pf(P, P, P, 1024, 8, 2, 128, 128, 4, P, ctypes.byref(L), None, P, None, WS, 1 << 30, None) == INVALID
    # workspace too small for one window of partials
    assert pf(P, P, P, 1024, 8, 2, 128, 128, 4, P, ctypes.byref(L), P2, P, None, WS, 1024, None) == WORKSPACE
    dec = msa.lib.msa_sparse_decode
    args = [P, P, P, P, P, P, 4, 4096, 64, 4, 128, 64, 128, 16, P, None, None, WS, 1 << 30, None]
    bad = list(args)
    bad[5] = None                                                # lens missing
    assert dec(*bad) == INVALID
    g32 = list(args)
    g32[8] = 128                                                 # G = 32 > 16 for decode
    assert dec(*g32) == UNSUPPORTED
    small = list(args)
    small[18] = 256
    assert dec(*small) == WORKSPACE


def test_host_fault_injection():
    """MSA_FAULT_INJECT=<entry point> makes that call fail as a launch failure would, before enqueueing."""
    code = (
        "import sys; sys.path.insert(0, %r)\n"
        "import block_sparse_long_idx_b200 as m\n"
        "r = m.lib.msa_index_topk(%d, %d, 1024, 2, 64, 128, 4, %d, %d, 256, None)\n"
        "print('STATUS', r)\n" % (ROOT, P, P2, P, WS))
    env = dict(os.environ, MSA_FAULT_INJECT="msa_index_topk")
    out = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=300)
    assert "STATUS 4" in out.stdout, out.stdout + out.stderr
    # the backward's injection point sits after its argument checks, before anything is enqueued
    code = (
        "import sys; sys.path.insert(0, %r)\n"
        "import block_sparse_long_idx_b200 as m\n"
        "r = m.lib.msa_sparse_backward(%d, %d, %d, %d, %d, %d, 1024, 8, 2, 64, 128, 4, %d, None, None, %d, %d, %d, "
        "None, None, 0, 1.0, None, None, None, %d, 1 << 40, None)\n"
        "print('STATUS', r)\n" % (ROOT, P, P, P, P, P2, P, P, P, P, P, WS))
    env = dict(os.environ, MSA_FAULT_INJECT="msa_sparse_backward")
    out = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=300)
    assert "STATUS 4" in out.stdout, out.stdout + out.stderr


def test_selftest_validation(msa):
    """The failure-path self-test rejects bad arguments before launching anything."""
    lib = msa.lib
    assert lib.msa_selftest_workspace_size() >= 8
    assert lib.msa_selftest_wait_timeout(None, 256, 1000, None) == INVALID
    assert lib.msa_selftest_wait_timeout(WS + 8, 256, 1000, None) == INVALID  # not 256-byte aligned
    assert lib.msa_selftest_wait_timeout(WS, 256, 0, None) == INVALID
    assert lib.msa_selftest_wait_timeout(WS, 256, 2_000_000_001, None) == INVALID
    assert lib.msa_selftest_wait_timeout(WS, 8, 1000, None) == WORKSPACE


def test_varlen_validation_and_sizes(msa):
    """Packed-batch prefill: cu_seqlens checks and workspace sizing happen on the host."""
    lib = msa.lib
    c_vp = ctypes.c_void_p
    import numpy as np

    def cu(*x):
        a = np.asarray(x, dtype=np.int32)
        return a, a.ctypes.data_as(c_vp)

    good, gp = cu(0, 100, 100, 1000, 4096)
    sz = lib.msa_sparse_prefill_varlen_workspace_size(gp, None, 4, 16, 2, 128, 128, 8, 0)
    assert sz > 0
    # fewer rows per pass -> smaller workspace, never below one window
    assert 0 < lib.msa_sparse_prefill_varlen_workspace_size(gp, None, 4, 16, 2, 128, 128, 8, 2048) <= sz
    for bad in ((1, 100), (0, 50, 40), (0, 0)):
        b, bp = cu(*bad)
        assert lib.msa_sparse_prefill_varlen_workspace_size(bp, None, len(bad) - 1, 16, 2, 128, 128, 8, 0) == 0
        assert lib.msa_sparse_prefill_varlen(P, P, P, P, P, bp, None, len(bad) - 1, 16, 2, 128, 64, 128, 8, P2, P,
                                             None, WS, sz, None) == INVALID
    args = (P, P, P, P, P, gp, None, 4, 16, 2, 128, 64, 128, 8, P2, P, None, WS)
    assert lib.msa_sparse_prefill_varlen(*args, 256, None) == WORKSPACE
    assert lib.msa_sparse_prefill_varlen(P, P, P, P, P, gp, None, 4, 16, 2, 96, 64, 128, 8, P2, P, None, WS, sz,
                                         None) == UNSUPPORTED
    assert lib.msa_sparse_prefill_varlen(P + 8, P, P, P, P, gp, None, 4, 16, 2, 128, 64, 128, 8, P2, P, None, WS, sz,
                                         None) == INVALID
    # keys with cached prefixes: whole blocks only, never fewer keys than queries
    ok_k, okp = cu(0, 228, 356, 1256, 4352)      # prefixes 128, 128, 0, 0 ... per sequence differences
    assert lib.msa_sparse_prefill_varlen_workspace_size(gp, okp, 4, 16, 2, 128, 128, 8, 0) > 0
    part, pp = cu(0, 150, 150, 1050, 4146)       # prefix 50: not a whole block
    assert lib.msa_sparse_prefill_varlen(P, P, P, P, P, gp, pp, 4, 16, 2, 128, 64, 128, 8, P2, P, None, WS, sz,
                                         None) == UNSUPPORTED
    short, sp = cu(0, 50, 50, 950, 4042)         # fewer keys than queries
    assert lib.msa_sparse_prefill_varlen(P, P, P, P, P, gp, sp, 4, 16, 2, 128, 64, 128, 8, P2, P, None, WS, sz,
                                         None) == INVALID


def test_missing_library_fails_loudly(tmp_path):
    """Without the built CUDA library the package refuses to load: there is no CPU or PyTorch path."""
    pkg = os.path.join(ROOT, "block_sparse_long_idx_b200")
    code = (
        "import sys, os, shutil\n"
        "sys.path.insert(0, %r)\n"
        "shutil.copytree(%r, os.path.join(%r, 'block_sparse_long_idx_b200'),\n"
        "                ignore=shutil.ignore_patterns('*.so', '_build', '__pycache__'))\n"
        "import block_sparse_long_idx_b200 as m\n"
        "try:\n"
        "    m.msa_index_topk\n"
        "except ImportError as e:\n"
        "    print('IMPORT_ERROR', 'no CPU or PyTorch fallback' in str(e))\n"
        "else:\n"
        "    print('LOADED')\n" % (str(tmp_path), pkg, str(tmp_path)))
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300,
                         cwd=str(tmp_path))
    assert "IMPORT_ERROR True" in out.stdout, out.stdout + out.stderr


def test_varlen_workspace_sizes_follow_the_batch(msa):
    """Workspace sizing of the packed-batch prefill: empty sequences are accepted, adding tokens or
    cached prefixes never shrinks the workspace, and a batch of one sequence needs at least the
    single-sequence prefill workspace."""
    import numpy as np

    lib = msa.lib
    c_vp = ctypes.c_void_p

    def size(cu, cuk=None, rows=0):
        a = np.asarray(cu, dtype=np.int32)
        b = None if cuk is None else np.asarray(cuk, dtype=np.int32)
        return lib.msa_sparse_prefill_varlen_workspace_size(
            a.ctypes.data_as(c_vp), None if b is None else b.ctypes.data_as(c_vp), len(cu) - 1, 16, 2, 128, 128, 8,
            rows)

    base = size([0, 1000, 3000])
    assert base > 0
    assert size([0, 0, 1000, 1000, 3000]) >= base > 0          # empty sequences
    assert size([0, 1000, 5000]) > base                        # more tokens
    assert size([0, 1000, 3000], [0, 1256, 3256]) >= base      # cached prefixes (256 each) add key blocks
    single = lib.msa_sparse_prefill_workspace_size(3000, 16, 2, 128, 128, 8, 0, 1)
    assert size([0, 3000]) >= single


def test_backward_validation_and_sizes(msa):
    f = msa.lib.msa_sparse_backward
    sz = msa.lib.msa_sparse_backward_workspace_size
    N, H_q, H_kv, d_h, k = 1024, 8, 2, 64, 4
    need = sz(N, H_q, H_kv, d_h, 128, k, 0, 0)
    assert need >= 4 * N * d_h * (H_q + 2 * H_kv) + 4 * N * H_q
    assert sz(N, H_q, H_kv, d_h, 128, k, 0, 1) > need                 # room for an internal inversion
    assert sz(N, H_q, H_kv, d_h, 128, k, 64, 0) >= need + 4 * N * H_kv * (2 * 64 + 1)  # KL accumulators
    assert sz(N, H_q, H_kv, d_h, 64, k, 0, 0) == 0                    # rejected shape
    assert sz(N, H_q, H_kv, d_h, 128, k, 48, 0) == 0                  # rejected d_idx
    ok = [P, P, P, P, P2, P, N, H_q, H_kv, d_h, 128, k, P, None, None, P, P, P, None, None, 0, 1.0, None, None, None,
          WS, 1 << 40, None]
    names = ["q", "k", "v", "out", "lse", "dout", "N", "H_q", "H_kv", "d_h", "B_k", "kk", "block_idx", "layout",
             "kv2q", "dq", "dk", "dv", "q_idx", "k_idx", "d_idx", "kl_weight", "dq_idx", "dk_idx", "kl", "ws",
             "ws_bytes", "stream"]

    def call(**kw):
        a = list(ok)
        for n, x in kw.items():
            a[names.index(n)] = x
        return f(*a)

    assert call(lse=None) == INVALID                  # the forward's lse is required
    assert call(dout=None) == INVALID
    assert call(block_idx=None) == INVALID            # neither selections nor an inversion
    assert call(dq=P + 8) == INVALID                  # misaligned output
    assert call(H_kv=3) == INVALID                    # H_q % H_kv
    assert call(H_q=64, H_kv=2) == UNSUPPORTED        # G = 32
    assert call(d_h=96) == UNSUPPORTED
    assert call(kk=17) == UNSUPPORTED
    assert call(ws_bytes=need - 1) == WORKSPACE
    kl = dict(q_idx=P, k_idx=P, d_idx=64, dq_idx=P, dk_idx=P, kl=P2)
    assert call(**dict(kl, dk_idx=None)) == INVALID      # KL outputs required with q_idx
    assert call(**dict(kl, block_idx=None)) == INVALID   # the KL part reads the selections
    assert call(**dict(kl, k_idx=P + 2)) == INVALID      # misaligned
    assert call(**dict(kl, d_idx=128)) == UNSUPPORTED
    assert call(**dict(kl, ws_bytes=need)) == WORKSPACE  # no room for the KL accumulators


def test_static_kv2q_validation(msa):
    """msa_build_kv2q_static validates the layout like msa_build_kv2q (every field, nb and n_windows
    included) and rejects it on the host before touching the device."""
    f = msa.lib.msa_build_kv2q_static
    L = msa.msa_kv2q_layout_get(5000, 2, 128, 16)
    assert f(None, ctypes.byref(L), P, None) == INVALID
    assert f(P, ctypes.byref(L), None, None) == INVALID
    assert f(P, ctypes.byref(L), P + 16, None) == INVALID       # kv2q buffer not 256-byte aligned
    for field, delta in (("nb", 1), ("n_windows", 1), ("max_items", 1), ("total_bytes", 256), ("entries", 256)):
        bad = msa.msa_kv2q_layout_get(5000, 2, 128, 16)
        setattr(bad, field, getattr(bad, field) + delta)
        assert f(P, ctypes.byref(bad), P2, None) == INVALID, field


def test_static_kv2q_fault_injection():
    """The host fault hook covers msa_build_kv2q_static too (fails before anything is enqueued)."""
    code = (
        "import sys, ctypes; sys.path.insert(0, %r)\n"
        "import block_sparse_long_idx_b200 as m\n"
        "L = m.msa_kv2q_layout_get(5000, 2, 128, 16)\n"
        "r = m.lib.msa_build_kv2q_static(%d, ctypes.byref(L), %d, None)\n"
        "print('STATUS', r)\n" % (ROOT, P, P2))
    env = dict(os.environ, MSA_FAULT_INJECT="msa_build_kv2q_static")
    out = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=300)
    assert "STATUS 4" in out.stdout, out.stdout + out.stderr
