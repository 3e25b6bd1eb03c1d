"""CPU oracle for the MSA forward path and its backward (test infrastructure only).

Only the tests, the package smoke check and the benchmark's CPU-baseline leg may import this
package. It wraps the plain C99 + OpenMP oracle in ``msa_oracle.c`` with numpy marshalling.
See ``msa_oracle.c`` for what each function computes and which passage it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "msa_oracle.c")
LIB = os.path.join(_HERE, "libmsa_oracle.so")

_c_u16p = ctypes.POINTER(ctypes.c_uint16)
_c_i32p = ctypes.POINTER(ctypes.c_int32)
_c_i64p = ctypes.POINTER(ctypes.c_int64)
_c_f64p = ctypes.POINTER(ctypes.c_double)
_int, _i64 = ctypes.c_int, ctypes.c_int64


def compile_oracle(src: str = SRC, out: str = LIB, force: bool = False) -> str:
    """Compile an oracle source with gcc (-O3, no FMA contraction, OpenMP) into a shared library."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        cmd = ["gcc", "-O3", "-march=x86-64-v2", "-ffp-contract=off", "-fopenmp", "-shared", "-fPIC",
               "-o", out + ".tmp", src, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(out + ".tmp", out)
    return out


def build(force: bool = False) -> str:
    return compile_oracle(SRC, LIB, force)


def _p(a: np.ndarray, t):
    return a.ctypes.data_as(t)


def _u16(a):
    return np.ascontiguousarray(a, dtype=np.uint16)


class Oracle:
    """numpy front end of one compiled oracle library."""

    def __init__(self, so_path: str):
        L = ctypes.CDLL(so_path)
        L.msa_oracle_select_rows.argtypes = [_c_u16p, _c_i64p, _i64, _c_u16p, _i64, _int, _int, _int, _int, _c_i32p,
                                             _int]
        L.msa_oracle_kv2q.argtypes = [_c_i32p, _i64, _int, _int, _int, _c_i64p, _c_i32p]
        L.msa_oracle_attend_rows.argtypes = [_c_u16p, _c_i64p, _i64, _c_u16p, _c_u16p, _i64, _int, _int, _int, _int,
                                             _int, _c_i32p, _c_f64p, _c_f64p, _int]
        L.msa_oracle_decode.argtypes = [_c_u16p, _c_u16p, _c_u16p, _c_u16p, _c_u16p, _c_i32p, _int, _i64, _int, _int,
                                        _int, _int, _int, _int, _c_f64p, _c_f64p, _c_i32p, _int]
        L.msa_oracle_backward_dq_rows.argtypes = [_c_u16p, _c_u16p, _c_i64p, _i64, _c_u16p, _c_u16p, _i64, _int, _int,
                                                  _int, _int, _int, _c_i32p, _c_f64p, _int]
        L.msa_oracle_backward_dkv_blocks.argtypes = [_c_u16p, _c_u16p, _c_u16p, _c_u16p, _i64, _int, _int, _int, _int,
                                                     _int, _c_i32p, _c_i32p, _i64, _c_f64p, _c_f64p, _int]
        L.msa_oracle_kl_rows.argtypes = [_c_u16p, _c_u16p, _c_i64p, _i64, _c_u16p, _c_u16p, _i64, _int, _int, _int,
                                         _int, _int, _int, _c_i32p, ctypes.c_double, _c_f64p, _c_f64p, _int]
        _c_u8p = ctypes.POINTER(ctypes.c_uint8)
        L.msa_oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.msa_oracle_e4m3_decode.restype = ctypes.c_double
        L.msa_oracle_e4m3_encode.argtypes = [ctypes.c_double]
        L.msa_oracle_e4m3_encode.restype = ctypes.c_uint8
        L.msa_oracle_quantize_e4m3_rows.argtypes = [_c_u16p, _i64, _int, _c_u8p, _c_f64p]
        L.msa_oracle_attend_rows_e4m3.argtypes = [_c_u8p, _c_f64p, _c_i64p, _i64, _c_u8p, _c_f64p, _c_u8p, _c_f64p,
                                                  _i64, _int, _int, _int, _int, _int, _c_i32p, _c_f64p, _c_f64p,
                                                  _int]
        L.msa_oracle_kl_dk_idx_blocks.argtypes = [_c_u16p, _c_u16p, _c_u16p, _c_u16p, _i64, _int, _int, _int, _int,
                                                  _int, _int, _c_i32p, _c_i32p, _i64, ctypes.c_double, _c_f64p, _int]
        for f in ("msa_oracle_select_rows", "msa_oracle_kv2q", "msa_oracle_attend_rows", "msa_oracle_decode",
                  "msa_oracle_max_threads", "msa_oracle_backward_dq_rows", "msa_oracle_backward_dkv_blocks",
                  "msa_oracle_kl_rows", "msa_oracle_kl_dk_idx_blocks", "msa_oracle_quantize_e4m3_rows",
                  "msa_oracle_attend_rows_e4m3"):
            getattr(L, f).restype = _int
        self.L = L

    def max_threads(self) -> int:
        return int(self.L.msa_oracle_max_threads())

    def select_rows(self, q_idx, k_idx, rows, B_k: int, k: int, n_threads: int = 0) -> np.ndarray:
        """Block selection for query rows.

        q_idx, k_idx: [N, H_kv, d_idx] bf16 bits. rows: positions. Returns int32 [len(rows), H_kv, k]."""
        N, H_kv, d_idx = k_idx.shape
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        qg = _u16(q_idx[rows])
        kk = _u16(k_idx)
        sel = np.empty((len(rows), H_kv, k), dtype=np.int32)
        rc = self.L.msa_oracle_select_rows(_p(qg, _c_u16p), _p(rows, _c_i64p), len(rows), _p(kk, _c_u16p), N, H_kv,
                                           d_idx, B_k, k, _p(sel, _c_i32p), n_threads)
        if rc:
            raise ValueError("msa_oracle_select_rows: bad arguments")
        return sel

    def select_all(self, q_idx, k_idx, B_k: int, k: int, n_threads: int = 0) -> np.ndarray:
        """Selections for every row, laid out [H_kv, N, k] like the library's block_idx."""
        N = k_idx.shape[0]
        sel = self.select_rows(q_idx, k_idx, np.arange(N), B_k, k, n_threads)
        return np.ascontiguousarray(sel.transpose(1, 0, 2))

    def kv2q(self, block_idx, B_k: int):
        """CSR inversion. block_idx [H_kv, N, k] -> (offsets int64 [H_kv, nb+1], per-group entry arrays)."""
        H_kv, N, k = block_idx.shape
        nb = (N + B_k - 1) // B_k
        bi = np.ascontiguousarray(block_idx, dtype=np.int32)
        off = np.zeros((H_kv, nb + 1), dtype=np.int64)
        ent = np.empty((H_kv, N * k), dtype=np.int32)
        rc = self.L.msa_oracle_kv2q(_p(bi, _c_i32p), N, H_kv, B_k, k, _p(off, _c_i64p), _p(ent, _c_i32p))
        if rc:
            raise ValueError("msa_oracle_kv2q: block id out of range")
        return off, [ent[r, : off[r, -1]].copy() for r in range(H_kv)]

    def attend_rows(self, q, kk, v, rows, sel, B_k: int, n_threads: int = 0):
        """Sparse attention for rows with selections sel [len(rows), H_kv, k].

        q [N, H_q, d_h], kk/v [N, H_kv, d_h] bf16 bits. Returns (out f64 [n, H_q, d_h], lse f64 [n, H_q])."""
        N, H_kv, d_h = kk.shape
        H_q = q.shape[1]
        k = sel.shape[2]
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        qg = _u16(q[rows])
        kc, vc = _u16(kk), _u16(v)
        sel = np.ascontiguousarray(sel, dtype=np.int32)
        out = np.empty((len(rows), H_q, d_h), dtype=np.float64)
        lse = np.empty((len(rows), H_q), dtype=np.float64)
        rc = self.L.msa_oracle_attend_rows(_p(qg, _c_u16p), _p(rows, _c_i64p), len(rows), _p(kc, _c_u16p),
                                           _p(vc, _c_u16p), N, H_q, H_kv, d_h, B_k, k, _p(sel, _c_i32p),
                                           _p(out, _c_f64p), _p(lse, _c_f64p), n_threads)
        if rc:
            raise ValueError("msa_oracle_attend_rows: bad arguments")
        return out, lse

    def prefill_rows(self, inputs: dict, rows, B_k: int, k: int, n_threads: int = 0):
        """Selection then attention for the given rows. Returns (sel [n, H_kv, k], out, lse)."""
        sel = self.select_rows(inputs["q_idx"], inputs["k_idx"], rows, B_k, k, n_threads)
        out, lse = self.attend_rows(inputs["q"], inputs["k"], inputs["v"], rows, sel, B_k, n_threads)
        return sel, out, lse

    def prefill_varlen_rows(self, inputs: dict, cu_seqlens, rows, B_k: int, k: int, n_threads: int = 0,
                            cu_seqlens_k=None):
        """Packed batch of independent sequences: query rows packed by cu_seqlens [B+1] (q, q_idx),
        keys packed by cu_seqlens_k [B+1] (k, v, k_idx; default: like the queries). A sequence with
        more keys than queries holds a cached prefix: its query rows are its last positions. Each
        sequence is its own causal problem, so each row is answered by the single-sequence path on
        that sequence's tokens (query rows placed at their positions), in the sequence's local block
        indices. Returns (sel [n, H_kv, k], out, lse) for the given global query rows."""
        cu = np.asarray(cu_seqlens, dtype=np.int64)
        cuk = cu if cu_seqlens_k is None else np.asarray(cu_seqlens_k, dtype=np.int64)
        rows = np.asarray(rows, dtype=np.int64)
        seq = np.searchsorted(cu, rows, side="right") - 1
        H_kv = inputs["k_idx"].shape[1]
        H_q, d_h = inputs["q"].shape[1], inputs["q"].shape[2]
        sel = np.empty((len(rows), H_kv, k), dtype=np.int32)
        out = np.empty((len(rows), H_q, d_h), dtype=np.float64)
        lse = np.empty((len(rows), H_q), dtype=np.float64)
        for s in np.unique(seq):
            lo, hi = int(cu[s]), int(cu[s + 1])
            klo, khi = int(cuk[s]), int(cuk[s + 1])
            prefix = (khi - klo) - (hi - lo)
            part = {n: np.ascontiguousarray(inputs[n][klo:khi]) for n in ("k", "v", "k_idx")}
            for n in ("q", "q_idx"):  # query rows at their positions; cached positions are never queried
                full = np.zeros((khi - klo,) + inputs[n].shape[1:], dtype=inputs[n].dtype)
                full[prefix:] = inputs[n][lo:hi]
                part[n] = full
            pick = np.nonzero(seq == s)[0]
            s_sel, s_out, s_lse = self.prefill_rows(part, rows[pick] - lo + prefix, B_k, k, n_threads)
            sel[pick], out[pick], lse[pick] = s_sel, s_out, s_lse
        return sel, out, lse

    def decode(self, inputs: dict, B_k: int, k: int, n_threads: int = 0):
        """Decode oracle. Returns (sel [B, H_kv, k], out f64 [B, H_q, d_h], lse f64 [B, H_q])."""
        q, qi = _u16(inputs["q"]), _u16(inputs["q_idx"])
        kc, vc, kic = _u16(inputs["k_cache"]), _u16(inputs["v_cache"]), _u16(inputs["k_idx_cache"])
        lens = np.ascontiguousarray(inputs["lens"], dtype=np.int32)
        B, H_q, d_h = q.shape
        L_max, H_kv = kc.shape[1], kc.shape[2]
        d_idx = qi.shape[2]
        out = np.empty((B, H_q, d_h), dtype=np.float64)
        lse = np.empty((B, H_q), dtype=np.float64)
        sel = np.empty((B, H_kv, k), dtype=np.int32)
        rc = self.L.msa_oracle_decode(_p(q, _c_u16p), _p(qi, _c_u16p), _p(kc, _c_u16p), _p(vc, _c_u16p),
                                      _p(kic, _c_u16p), _p(lens, _c_i32p), B, L_max, H_q, H_kv, d_h, d_idx, B_k, k,
                                      _p(out, _c_f64p), _p(lse, _c_f64p), _p(sel, _c_i32p), n_threads)
        if rc:
            raise ValueError("msa_oracle_decode: bad arguments")
        return sel, out, lse

    # ------------------------------------------------------------------ backward
    def backward_dq_rows(self, q, dout, kk, v, rows, sel, B_k: int, n_threads: int = 0) -> np.ndarray:
        """Main-branch dq of the given rows (selections sel [len(rows), H_kv, k] held fixed).

        q, dout [N, H_q, d_h], kk/v [N, H_kv, d_h] bf16 bits. Returns f64 [len(rows), H_q, d_h]."""
        N, H_kv, d_h = kk.shape
        H_q = q.shape[1]
        k = sel.shape[2]
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        qg, dg = _u16(q[rows]), _u16(dout[rows])
        kc, vc = _u16(kk), _u16(v)
        sel = np.ascontiguousarray(sel, dtype=np.int32)
        dq = np.empty((len(rows), H_q, d_h), dtype=np.float64)
        rc = self.L.msa_oracle_backward_dq_rows(_p(qg, _c_u16p), _p(dg, _c_u16p), _p(rows, _c_i64p), len(rows),
                                                _p(kc, _c_u16p), _p(vc, _c_u16p), N, H_q, H_kv, d_h, B_k, k,
                                                _p(sel, _c_i32p), _p(dq, _c_f64p), n_threads)
        if rc:
            raise ValueError("msa_oracle_backward_dq_rows: bad arguments")
        return dq

    def backward_dkv_blocks(self, q, dout, kk, v, sel, pairs, B_k: int, n_threads: int = 0):
        """Main-branch dk, dv of whole KV blocks. sel [N, H_kv, k]: selections of every row;
        pairs [(r, b), ...]. Returns (dk, dv) f64 [len(pairs), B_k, d_h] (rows past N are zero)."""
        N, H_kv, d_h = kk.shape
        H_q = q.shape[1]
        k = sel.shape[2]
        qc, dc, kc, vc = _u16(q), _u16(dout), _u16(kk), _u16(v)
        sel = np.ascontiguousarray(sel, dtype=np.int32)
        pr = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32).reshape(-1, 2))
        dk = np.empty((len(pr), B_k, d_h), dtype=np.float64)
        dv = np.empty((len(pr), B_k, d_h), dtype=np.float64)
        rc = self.L.msa_oracle_backward_dkv_blocks(_p(qc, _c_u16p), _p(dc, _c_u16p), _p(kc, _c_u16p), _p(vc, _c_u16p),
                                                   N, H_q, H_kv, d_h, B_k, k, _p(sel, _c_i32p), _p(pr, _c_i32p),
                                                   len(pr), _p(dk, _c_f64p), _p(dv, _c_f64p), n_threads)
        if rc:
            raise ValueError("msa_oracle_backward_dkv_blocks: bad arguments")
        return dk, dv

    def kl_rows(self, q, q_idx, kk, k_idx, rows, sel, B_k: int, w: float = 1.0, n_threads: int = 0):
        """Index-branch KL of the given rows and its gradient in q_idx (scaled by w).

        Returns (kl f64 [len(rows), H_kv], dq_idx f64 [len(rows), H_kv, d_idx])."""
        N, H_kv, d_h = kk.shape
        H_q, d_idx = q.shape[1], k_idx.shape[2]
        k = sel.shape[2]
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        qg, qig = _u16(q[rows]), _u16(q_idx[rows])
        kc, kic = _u16(kk), _u16(k_idx)
        sel = np.ascontiguousarray(sel, dtype=np.int32)
        kl = np.empty((len(rows), H_kv), dtype=np.float64)
        dq_idx = np.empty((len(rows), H_kv, d_idx), dtype=np.float64)
        rc = self.L.msa_oracle_kl_rows(_p(qg, _c_u16p), _p(qig, _c_u16p), _p(rows, _c_i64p), len(rows), _p(kc, _c_u16p),
                                       _p(kic, _c_u16p), N, H_q, H_kv, d_h, d_idx, B_k, k, _p(sel, _c_i32p), float(w),
                                       _p(kl, _c_f64p), _p(dq_idx, _c_f64p), n_threads)
        if rc:
            raise ValueError("msa_oracle_kl_rows: bad arguments")
        return kl, dq_idx

    def kl_dk_idx_blocks(self, q, q_idx, kk, k_idx, sel, pairs, B_k: int, w: float = 1.0, n_threads: int = 0):
        """Gradient of the index-branch KL in k_idx for whole KV blocks (scaled by w).
        sel [N, H_kv, k]: selections of every row. Returns f64 [len(pairs), B_k, d_idx]."""
        N, H_kv, d_h = kk.shape
        H_q, d_idx = q.shape[1], k_idx.shape[2]
        k = sel.shape[2]
        qc, qic, kc, kic = _u16(q), _u16(q_idx), _u16(kk), _u16(k_idx)
        sel = np.ascontiguousarray(sel, dtype=np.int32)
        pr = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32).reshape(-1, 2))
        g = np.empty((len(pr), B_k, d_idx), dtype=np.float64)
        rc = self.L.msa_oracle_kl_dk_idx_blocks(_p(qc, _c_u16p), _p(qic, _c_u16p), _p(kc, _c_u16p), _p(kic, _c_u16p), N,
                                                H_q, H_kv, d_h, d_idx, B_k, k, _p(sel, _c_i32p), _p(pr, _c_i32p),
                                                len(pr), float(w), _p(g, _c_f64p), n_threads)
        if rc:
            raise ValueError("msa_oracle_kl_dk_idx_blocks: bad arguments")
        return g

    # ------------------------------------------------------------------ FP8 (E4M3) main branch
    def e4m3_decode(self, code: int) -> float:
        return float(self.L.msa_oracle_e4m3_decode(code))

    def e4m3_encode(self, x: float) -> int:
        return int(self.L.msa_oracle_e4m3_encode(float(x)))

    def quantize_e4m3(self, x):
        """Per-row E4M3 quantisation of a bf16 tensor [..., cols]: (codes uint8 same shape, scales f64 [...])."""
        xs = _u16(x)
        rows = int(np.prod(xs.shape[:-1]))
        codes = np.empty(xs.shape, dtype=np.uint8)
        scales = np.empty(xs.shape[:-1], dtype=np.float64)
        rc = self.L.msa_oracle_quantize_e4m3_rows(_p(xs, _c_u16p), rows, xs.shape[-1],
                                                  codes.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)),
                                                  _p(scales, _c_f64p))
        if rc:
            raise ValueError("msa_oracle_quantize_e4m3_rows: bad arguments")
        return codes, scales

    def attend_rows_e4m3(self, q8, k8, v8, rows, sel, B_k: int, n_threads: int = 0):
        """Sparse attention on E4M3 inputs; q8/k8/v8 = (codes, scales) from quantize_e4m3 of q [N, H_q, d_h],
        k/v [N, H_kv, d_h]. Returns (out f64 [n, H_q, d_h], lse f64 [n, H_q])."""
        (qc, qs), (kc, ks), (vc, vs) = q8, k8, v8
        N, H_kv, d_h = kc.shape
        H_q = qc.shape[1]
        k = sel.shape[2]
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        u8 = ctypes.POINTER(ctypes.c_uint8)
        qg, qsg = np.ascontiguousarray(qc[rows]), np.ascontiguousarray(qs[rows])
        kc, ks, vc, vs = (np.ascontiguousarray(a) for a in (kc, ks, vc, vs))
        sel = np.ascontiguousarray(sel, dtype=np.int32)
        out = np.empty((len(rows), H_q, d_h), dtype=np.float64)
        lse = np.empty((len(rows), H_q), dtype=np.float64)
        rc = self.L.msa_oracle_attend_rows_e4m3(qg.ctypes.data_as(u8), _p(qsg, _c_f64p), _p(rows, _c_i64p), len(rows),
                                                kc.ctypes.data_as(u8), _p(ks, _c_f64p), vc.ctypes.data_as(u8),
                                                _p(vs, _c_f64p), N, H_q, H_kv, d_h, B_k, k, _p(sel, _c_i32p),
                                                _p(out, _c_f64p), _p(lse, _c_f64p), n_threads)
        if rc:
            raise ValueError("msa_oracle_attend_rows_e4m3: bad arguments")
        return out, lse


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def select_rows(*a, **kw):
    return default().select_rows(*a, **kw)


def select_all(*a, **kw):
    return default().select_all(*a, **kw)


def kv2q(*a, **kw):
    return default().kv2q(*a, **kw)


def attend_rows(*a, **kw):
    return default().attend_rows(*a, **kw)


def prefill_rows(*a, **kw):
    return default().prefill_rows(*a, **kw)


def prefill_varlen_rows(*a, **kw):
    return default().prefill_varlen_rows(*a, **kw)


def decode(*a, **kw):
    return default().decode(*a, **kw)


def backward_dq_rows(*a, **kw):
    return default().backward_dq_rows(*a, **kw)


def backward_dkv_blocks(*a, **kw):
    return default().backward_dkv_blocks(*a, **kw)


def kl_rows(*a, **kw):
    return default().kl_rows(*a, **kw)


def kl_dk_idx_blocks(*a, **kw):
    return default().kl_dk_idx_blocks(*a, **kw)


def quantize_e4m3(*a, **kw):
    return default().quantize_e4m3(*a, **kw)


def attend_rows_e4m3(*a, **kw):
    return default().attend_rows_e4m3(*a, **kw)


def max_threads() -> int:
    return default().max_threads()
