"""Python binding of libmsa_b200.so, the B200 (sm_100a) MiniMax Sparse Attention forward path.

Argument marshalling only: every step of the path runs in the library's CUDA kernels. Tensors are
torch CUDA tensors (bf16 data may be passed as torch.bfloat16 or as 16-bit integer bit patterns);
the current torch CUDA stream is used unless one is given. Functions keep the C names.

If the compiled library is missing the import fails loudly: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmsa_b200.so")

MSA_OK = 0
STATUS_NAMES = {0: "MSA_OK", 1: "MSA_ERR_INVALID_ARG", 2: "MSA_ERR_UNSUPPORTED", 3: "MSA_ERR_WORKSPACE",
                4: "MSA_ERR_CUDA", 5: "MSA_ERR_TIMEOUT", 6: "MSA_ERR_DEVICE_CHECK"}


class MsaError(RuntimeError):
    def __init__(self, fn: str, status: int, detail: str = ""):
        super().__init__(f"{fn}: {STATUS_NAMES.get(status, status)}" + (f" [{detail}]" if detail else ""))
        self.status = status


class msa_kv2q_layout(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("H_kv", ctypes.c_int32), ("B_k", ctypes.c_int32), ("k", ctypes.c_int32),
                ("nb", ctypes.c_int32), ("window", ctypes.c_int32), ("chunk", ctypes.c_int32),
                ("n_windows", ctypes.c_int32), ("max_items", ctypes.c_int64), ("offsets", ctypes.c_size_t),
                ("entries", ctypes.c_size_t), ("items", ctypes.c_size_t), ("window_items", ctypes.c_size_t),
                ("counts", ctypes.c_size_t), ("bases", ctypes.c_size_t), ("total_bytes", ctypes.c_size_t)]


_vp, _i64, _int, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
_LP = ctypes.POINTER(msa_kv2q_layout)

# (name, restype, argtypes) for every symbol declared in include/msa.h
SIGNATURES = [
    ("msa_status_string", ctypes.c_char_p, [_int]),
    ("msa_get_device_error", _int, [_vp, _vp]),
    ("msa_index_topk_workspace_size", _sz, [_i64, _int, _int, _int, _int]),
    ("msa_index_topk", _int, [_vp, _vp, _i64, _int, _int, _int, _int, _vp, _vp, _sz, _vp]),
    ("msa_kv2q_layout_get", _int, [_i64, _int, _int, _int, _int, _int, _LP]),
    ("msa_build_kv2q_workspace_size", _sz, [_LP]),
    ("msa_build_kv2q", _int, [_vp, _LP, _vp, _vp, _sz, _vp]),
    ("msa_build_kv2q_static", _int, [_vp, _LP, _vp, _vp]),
    ("msa_sparse_prefill_workspace_size", _sz, [_i64, _int, _int, _int, _int, _int, _i64, _int]),
    ("msa_sparse_prefill", _int, [_vp, _vp, _vp, _i64, _int, _int, _int, _int, _int, _vp, _LP, _vp, _vp, _vp, _vp,
                                  _sz, _vp]),
    ("msa_sparse_decode_workspace_size", _sz, [_int, _i64, _int, _int, _int, _int, _int, _int]),
    ("msa_sparse_decode", _int, [_vp, _vp, _vp, _vp, _vp, _vp, _int, _i64, _int, _int, _int, _int, _int, _int, _vp,
                                 _vp, _vp, _vp, _sz, _vp]),
    ("msa_sparse_prefill_varlen_workspace_size", _sz, [_vp, _vp, _int, _int, _int, _int, _int, _int, _i64]),
    ("msa_sparse_prefill_varlen", _int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _int, _int, _int, _int, _int, _int, _int,
                                         _vp, _vp, _vp, _vp, _sz, _vp]),
    ("msa_sparse_backward_workspace_size", _sz, [_i64, _int, _int, _int, _int, _int, _int, _int]),
    ("msa_sparse_backward", _int, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _int, _int, _int, _int, _int, _vp, _LP, _vp,
                                   _vp, _vp, _vp, _vp, _vp, _int, ctypes.c_float, _vp, _vp, _vp, _vp, _sz, _vp]),
    ("msa_quantize_e4m3", _int, [_vp, _i64, _int, _int, _vp, _vp, _vp, _vp, _vp]),
    ("msa_sparse_prefill_fp8", _int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _int, _int, _int, _int, _int,
                                      _vp, _LP, _vp, _vp, _vp, _vp, _sz, _vp]),
    ("msa_selftest_workspace_size", _sz, []),
    ("msa_selftest_wait_timeout", _int, [_vp, _sz, _i64, _vp]),
    ("msa_trace_set", None, [_vp]),
    ("msa_last_error_string", ctypes.c_char_p, []),
    ("msa_launch_count", ctypes.c_uint64, []),
]

KERNEL_NAMES = {1: "index_topk", 2: "kv2q", 3: "attn", 4: "combine", 5: "dec_pool", 6: "dec_topk", 7: "dec_attn",
                8: "dec_combine", 9: "bwd_prep", 10: "bwd_attn", 11: "bwd_convert", 12: "quant"}


class msa_trace(ctypes.Structure):
    _fields_ = [("events", ctypes.POINTER(ctypes.c_void_p)), ("capacity", ctypes.c_int), ("count", ctypes.c_int),
                ("kernel_ids", ctypes.POINTER(ctypes.c_int))]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m block_sparse_long_idx_b200.build` "
                          "(there is no CPU or PyTorch fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, res, args in SIGNATURES:
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


lib = _load()


def _check(fn: str, status: int):
    if status != MSA_OK:
        detail = lib.msa_last_error_string().decode() if status == 4 else ""
        raise MsaError(fn, status, detail)


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _bf16(t, name):
    if not t.is_cuda or not t.is_contiguous() or t.element_size() != 2:
        raise ValueError(f"{name}: expected a contiguous 16-bit CUDA tensor")
    return t


def _workspace(nbytes: int, device, ws):
    if ws is None:
        return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
    if ws.numel() * ws.element_size() < nbytes:
        raise ValueError("workspace too small")
    return ws


def msa_launch_count() -> int:
    """Kernels launched by the library so far in this process."""
    return int(lib.msa_launch_count())


class KernelTrace:
    """Per-kernel CUDA-event timing of library calls made while active (``with KernelTrace(n) as t``).

    After the traced work has finished, ``t.durations()`` maps kernel name -> list of durations (ms)."""

    def __init__(self, max_kernels: int = 4096):
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(2 * max_kernels)]
        for e in self.events:  # torch creates the CUDA event lazily, at its first record
            e.record()
        torch.cuda.synchronize()
        self._handles = (ctypes.c_void_p * len(self.events))(*[e.cuda_event for e in self.events])
        self._ids = (ctypes.c_int * max_kernels)()
        self.rec = msa_trace(self._handles, len(self.events), 0, self._ids)

    def __enter__(self):
        self.rec.count = 0
        lib.msa_trace_set(ctypes.byref(self.rec))
        return self

    def __exit__(self, *exc):
        lib.msa_trace_set(None)
        return False

    def durations(self):
        torch.cuda.synchronize()
        out = {}
        for j in range(self.rec.count // 2):
            name = KERNEL_NAMES.get(self._ids[j], str(self._ids[j]))
            out.setdefault(name, []).append(self.events[2 * j].elapsed_time(self.events[2 * j + 1]))
        return out


def status_string(status: int) -> str:
    return lib.msa_status_string(status).decode()


def msa_get_device_error(workspace: torch.Tensor, stream=None) -> int:
    """Device error word of a workspace used by a previous call (synchronises the stream)."""
    return lib.msa_get_device_error(workspace.data_ptr(), _stream(stream))


def msa_sparse_prefill_varlen(q, k_, v, q_idx, k_idx, cu_seqlens, B_k: int = 128, k: int = 16, block_idx=None,
                              out=None, lse=None, want_lse: bool = True, workspace=None, max_rows_per_pass: int = 0,
                              stream=None, cu_seqlens_k=None):
    """Packed batch of independent sequences (cu_seqlens [B+1], host ints, over the query rows;
    cu_seqlens_k over the key rows when keys hold cached prefixes): index branch, inversion,
    attention and combine in one call. Returns (out [T, H_q, d_h], lse [T, H_q], block_idx [H_kv, T, k])."""
    for t, n in ((q, "q"), (k_, "k"), (v, "v"), (q_idx, "q_idx"), (k_idx, "k_idx")):
        _bf16(t, n)
    T, H_q, d_h = q.shape
    H_kv, d_idx = k_idx.shape[1], k_idx.shape[2]
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    B = len(cu) - 1
    cu_p = cu.ctypes.data_as(ctypes.c_void_p)
    cuk = None if cu_seqlens_k is None else np.ascontiguousarray(np.asarray(cu_seqlens_k, dtype=np.int32))
    cuk_p = None if cuk is None else cuk.ctypes.data_as(ctypes.c_void_p)
    if block_idx is None:
        block_idx = torch.empty((H_kv, T, k), dtype=torch.int32, device=q.device)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((T, H_q), dtype=torch.float32, device=q.device)
    need = lib.msa_sparse_prefill_varlen_workspace_size(cu_p, cuk_p, B, H_q, H_kv, d_h, B_k, k, max_rows_per_pass)
    if need == 0:
        raise MsaError("msa_sparse_prefill_varlen_workspace_size", 1, "arguments rejected")
    ws = _workspace(need, q.device, workspace)
    _check("msa_sparse_prefill_varlen", lib.msa_sparse_prefill_varlen(
        q.data_ptr(), k_.data_ptr(), v.data_ptr(), q_idx.data_ptr(), k_idx.data_ptr(), cu_p, cuk_p, B, H_q, H_kv, d_h,
        d_idx,
        B_k, k, block_idx.data_ptr(), out.data_ptr(), _ptr(lse), ws.data_ptr(), ws.numel(), _stream(stream)))
    return out, lse, block_idx


def msa_selftest_wait_timeout(limit_cycles: int = 1_000_000, workspace=None, device=None, stream=None) -> int:
    """Runs the bounded-wait failure path on the device (a wait that can never complete) and
    returns the device status it left: MSA_ERR_TIMEOUT when the path works."""
    dev = workspace.device if workspace is not None else (device or torch.device("cuda"))
    ws = _workspace(lib.msa_selftest_workspace_size(), dev, workspace)
    _check("msa_selftest_wait_timeout", lib.msa_selftest_wait_timeout(ws.data_ptr(), ws.numel(), int(limit_cycles),
                                                                       _stream(stream)))
    return msa_get_device_error(ws, stream)


def msa_index_topk(q_idx, k_idx, B_k: int = 128, k: int = 16, block_idx=None, workspace=None, stream=None):
    """Index Branch: scores, block max-pool, Top-k with forced local block. Returns block_idx [H_kv, N, k] int32."""
    _bf16(q_idx, "q_idx")
    _bf16(k_idx, "k_idx")
    N, H_kv, d_idx = k_idx.shape
    if block_idx is None:
        block_idx = torch.empty((H_kv, N, k), dtype=torch.int32, device=k_idx.device)
    ws = _workspace(lib.msa_index_topk_workspace_size(N, H_kv, d_idx, B_k, k), k_idx.device, workspace)
    _check("msa_index_topk", lib.msa_index_topk(q_idx.data_ptr(), k_idx.data_ptr(), N, H_kv, d_idx, B_k, k,
                                                 block_idx.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream)))
    return block_idx


def msa_kv2q_layout_get(N: int, H_kv: int, B_k: int = 128, k: int = 16, window: int = 0, chunk: int = 0):
    L = msa_kv2q_layout()
    _check("msa_kv2q_layout_get", lib.msa_kv2q_layout_get(N, H_kv, B_k, k, window, chunk, ctypes.byref(L)))
    return L


class KV2Q:
    """A built KV->Q inversion: the host layout plus the device buffer it describes."""

    def __init__(self, layout: msa_kv2q_layout, buf: torch.Tensor):
        self.layout = layout
        self.buf = buf

    def _i32(self, off: int, n: int) -> torch.Tensor:
        return self.buf[off: off + 4 * n].view(torch.int32)

    def offsets(self) -> torch.Tensor:
        L = self.layout
        return self._i32(L.offsets, L.H_kv * (L.nb + 1)).view(L.H_kv, L.nb + 1)

    def entries(self) -> torch.Tensor:
        L = self.layout
        return self._i32(L.entries, L.H_kv * L.N * L.k).view(L.H_kv, L.N * L.k)

    def window_items(self) -> torch.Tensor:
        L = self.layout
        return self._i32(L.window_items, L.n_windows + 1)

    def items(self, n: int) -> torch.Tensor:
        """First n work items as int32 [n, 4] = (r, b, start, len)."""
        return self._i32(self.layout.items, 4 * n).view(n, 4)


def msa_build_kv2q(block_idx, B_k: int = 128, window: int = 0, chunk: int = 0, workspace=None, stream=None) -> KV2Q:
    """KV->Q inversion of block_idx [H_kv, N, k] into per-block query lists and a work list."""
    H_kv, N, k = block_idx.shape
    L = msa_kv2q_layout_get(N, H_kv, B_k, k, window, chunk)
    buf = torch.empty(L.total_bytes, dtype=torch.uint8, device=block_idx.device)
    ws = _workspace(lib.msa_build_kv2q_workspace_size(ctypes.byref(L)), block_idx.device, workspace)
    _check("msa_build_kv2q", lib.msa_build_kv2q(block_idx.data_ptr(), ctypes.byref(L), buf.data_ptr(),
                                                 ws.data_ptr(), ws.numel(), _stream(stream)))
    return KV2Q(L, buf)


def msa_sparse_prefill_workspace_size(N, H_q, H_kv, d_h, B_k=128, k=16, max_rows_per_pass=0, internal_kv2q=False):
    return lib.msa_sparse_prefill_workspace_size(N, H_q, H_kv, d_h, B_k, k, max_rows_per_pass, int(internal_kv2q))


def msa_sparse_prefill(q, k_, v, block_idx, kv2q: KV2Q | None = None, B_k: int = 128, out=None, lse=None,
                       want_lse: bool = True, workspace=None, max_rows_per_pass: int = 0, stream=None):
    """Main Branch: exact block-sparse attention on the selected blocks. Returns (out, lse)."""
    for t, n in ((q, "q"), (k_, "k"), (v, "v")):
        _bf16(t, n)
    N, H_q, d_h = q.shape
    H_kv = k_.shape[1]
    kk = block_idx.shape[2]
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((N, H_q), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(msa_sparse_prefill_workspace_size(N, H_q, H_kv, d_h, B_k, kk, max_rows_per_pass,
                                                                  kv2q is None), dtype=torch.uint8, device=q.device)
    lp = ctypes.byref(kv2q.layout) if kv2q is not None else None
    _check("msa_sparse_prefill", lib.msa_sparse_prefill(
        q.data_ptr(), k_.data_ptr(), v.data_ptr(), N, H_q, H_kv, d_h, B_k, kk, block_idx.data_ptr(), lp,
        _ptr(kv2q.buf) if kv2q is not None else None, out.data_ptr(), _ptr(lse), workspace.data_ptr(),
        workspace.numel(), _stream(stream)))
    return out, lse


def msa_sparse_backward(q, k_, v, out, lse, dout, block_idx=None, kv2q: KV2Q | None = None, B_k: int = 128,
                        k: int | None = None, dq=None, dk=None, dv=None, q_idx=None, k_idx=None,
                        kl_weight: float = 1.0, want_kl: bool = True, workspace=None, stream=None):
    """Main-branch backward with the selections held fixed: gradients of sum(dout * out) in q, k, v.

    out, lse: the forward's results for the same q, k, v and selections. Returns (dq, dk, dv) bf16.
    With q_idx, k_idx (the index branch's inputs; needs block_idx) the same pass also returns the
    KL alignment's gradients and per-(row, group) KL: (dq, dk, dv, dq_idx, dk_idx, kl)."""
    for t, n in ((q, "q"), (k_, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _bf16(t, n)
    if not lse.is_cuda or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse: expected a contiguous float32 CUDA tensor")
    N, H_q, d_h = q.shape
    H_kv = k_.shape[1]
    if k is None:
        if block_idx is None:
            raise ValueError("msa_sparse_backward: k is needed when block_idx is not given")
        k = block_idx.shape[2]
    if kv2q is None and block_idx is None:
        raise ValueError("msa_sparse_backward: give block_idx or a built kv2q")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k_) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    with_kl = q_idx is not None
    d_idx = 0
    dq_idx = dk_idx = kl = None
    if with_kl:
        _bf16(q_idx, "q_idx")
        _bf16(k_idx, "k_idx")
        if block_idx is None:
            raise ValueError("msa_sparse_backward: the KL part needs block_idx")
        d_idx = q_idx.shape[2]
        dq_idx, dk_idx = torch.empty_like(q_idx), torch.empty_like(k_idx)
        kl = torch.empty((N, H_kv), dtype=torch.float32, device=q.device) if want_kl else None
    ws = _workspace(lib.msa_sparse_backward_workspace_size(N, H_q, H_kv, d_h, B_k, k, d_idx, kv2q is None),
                    q.device, workspace)
    lp = ctypes.byref(kv2q.layout) if kv2q is not None else None
    _check("msa_sparse_backward", lib.msa_sparse_backward(
        q.data_ptr(), k_.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), dout.data_ptr(), N, H_q, H_kv, d_h,
        B_k, k, _ptr(block_idx), lp, _ptr(kv2q.buf) if kv2q is not None else None, dq.data_ptr(), dk.data_ptr(),
        dv.data_ptr(), _ptr(q_idx), _ptr(k_idx), d_idx, float(kl_weight), _ptr(dq_idx), _ptr(dk_idx), _ptr(kl),
        ws.data_ptr(), ws.numel(), _stream(stream)))
    if with_kl:
        return dq, dk, dv, dq_idx, dk_idx, kl
    return dq, dk, dv


def msa_sparse_decode(q, q_idx, k_cache, v_cache, k_idx_cache, lens, B_k: int = 128, k: int = 16, out=None, lse=None,
                      want_lse: bool = True, block_idx_out=None, workspace=None, stream=None):
    """Decode: one query per sequence at position lens-1. Returns (out, lse, block_idx)."""
    for t, n in ((q, "q"), (q_idx, "q_idx"), (k_cache, "k_cache"), (v_cache, "v_cache"),
                 (k_idx_cache, "k_idx_cache")):
        _bf16(t, n)
    B, H_q, d_h = q.shape
    L_max, H_kv = k_cache.shape[1], k_cache.shape[2]
    d_idx = q_idx.shape[2]
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, H_q), dtype=torch.float32, device=q.device)
    if block_idx_out is None:
        block_idx_out = torch.empty((B, H_kv, k), dtype=torch.int32, device=q.device)
    ws = _workspace(lib.msa_sparse_decode_workspace_size(B, L_max, H_q, H_kv, d_h, d_idx, B_k, k), q.device,
                    workspace)
    _check("msa_sparse_decode", lib.msa_sparse_decode(
        q.data_ptr(), q_idx.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), k_idx_cache.data_ptr(),
        lens.data_ptr(), B, L_max, H_q, H_kv, d_h, d_idx, B_k, k, out.data_ptr(), _ptr(lse),
        block_idx_out.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream)))
    return out, lse, block_idx_out


class E4M3Rows:
    """Per-row E4M3 quantisation of a [N, H, d] tensor: codes [N, H, d] uint8, scales and rscales
    [H, S] float32 (S = N rounded up to whole 128-token blocks), blkmax [H, S / 128] float32."""

    def __init__(self, codes, scales, rscales, blkmax):
        self.codes, self.scales, self.rscales, self.blkmax = codes, scales, rscales, blkmax


def msa_quantize_e4m3(x, with_rscales: bool = True, with_blkmax: bool = True, stream=None) -> E4M3Rows:
    """E4M3 codes and per-row scales (amax / 448) of x [N, H, d] bf16."""
    _bf16(x, "x")
    N, H, d = x.shape
    S = (N + 127) // 128 * 128
    codes = torch.empty((N, H, d), dtype=torch.uint8, device=x.device)
    scales = torch.empty((H, S), dtype=torch.float32, device=x.device)
    rscales = torch.empty((H, S), dtype=torch.float32, device=x.device) if with_rscales else None
    blkmax = torch.empty((H, S // 128), dtype=torch.float32, device=x.device) if with_blkmax else None
    _check("msa_quantize_e4m3", lib.msa_quantize_e4m3(x.data_ptr(), N, H, d, codes.data_ptr(), scales.data_ptr(),
                                                       _ptr(rscales), _ptr(blkmax), _stream(stream)))
    return E4M3Rows(codes, scales, rscales, blkmax)


def msa_sparse_prefill_fp8(q8: E4M3Rows, k8: E4M3Rows, v8: E4M3Rows, block_idx, kv2q: KV2Q | None = None,
                           B_k: int = 128, out=None, lse=None, want_lse: bool = True, workspace=None,
                           max_rows_per_pass: int = 0, stream=None):
    """FP8 main branch on E4M3 codes and scales from msa_quantize_e4m3. Returns (out bf16, lse)."""
    N, H_q, d_h = q8.codes.shape
    H_kv = k8.codes.shape[1]
    kk = block_idx.shape[2]
    if out is None:
        out = torch.empty((N, H_q, d_h), dtype=torch.bfloat16, device=q8.codes.device)
    if lse is None and want_lse:
        lse = torch.empty((N, H_q), dtype=torch.float32, device=q8.codes.device)
    if workspace is None:
        workspace = torch.empty(msa_sparse_prefill_workspace_size(N, H_q, H_kv, d_h, B_k, kk, max_rows_per_pass,
                                                                  kv2q is None), dtype=torch.uint8,
                                device=q8.codes.device)
    lp = ctypes.byref(kv2q.layout) if kv2q is not None else None
    _check("msa_sparse_prefill_fp8", lib.msa_sparse_prefill_fp8(
        q8.codes.data_ptr(), q8.scales.data_ptr(), k8.codes.data_ptr(), k8.scales.data_ptr(), v8.codes.data_ptr(),
        v8.scales.data_ptr(), v8.rscales.data_ptr(), v8.blkmax.data_ptr(), N, H_q, H_kv, d_h, B_k, kk,
        block_idx.data_ptr(), lp, _ptr(kv2q.buf) if kv2q is not None else None, out.data_ptr(), _ptr(lse),
        workspace.data_ptr(), workspace.numel(), _stream(stream)))
    return out, lse
