"""Helpers shared by the GPU parity tests: host<->device transfer and comparison against the oracle."""
from __future__ import annotations

import numpy as np
import torch

# Tolerance stated for bf16 inputs with fp32 accumulation: outputs within max |d| <= 1e-2 and
# mean |d| <= 1e-3 of the fp64 oracle; lse (fp32 output) within 1e-3 absolute.
OUT_MAX_ABS = 1e-2
OUT_MEAN_ABS = 1e-3
LSE_MAX_ABS = 1e-3


def dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    """Host array -> CUDA tensor with the same bits (uint16 bf16 patterns become int16)."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(device)
    return torch.from_numpy(a).to(device)


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    """bf16 device tensor (or int16 bit patterns) -> float64 numpy."""
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    u = t.cpu().numpy().view(np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def assert_out_close(got: np.ndarray, want: np.ndarray, what: str = "out"):
    d = np.abs(got - want)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    mx, mean = float(d.max()), float(d.mean())
    assert mx <= OUT_MAX_ABS and mean <= OUT_MEAN_ABS, (
        f"{what}: max |d| = {mx:.3e} (<= {OUT_MAX_ABS}), mean |d| = {mean:.3e} (<= {OUT_MEAN_ABS}); "
        f"worst index {np.unravel_index(int(d.argmax()), d.shape)}")
    return mx, mean


class OutErr:
    """|got - want| over many chunks of one output: max and mean over every value, checked at the end
    against the same tolerance as assert_out_close."""

    def __init__(self, what: str = "out"):
        self.what, self.mx, self.total, self.n, self.worst = what, 0.0, 0.0, 0, None

    def update(self, got: np.ndarray, want: np.ndarray, offset=0):
        assert np.isfinite(got).all(), f"{self.what}: non-finite values"
        d = np.abs(got - want)
        m = float(d.max())
        if m > self.mx:
            idx = np.unravel_index(int(d.argmax()), d.shape)
            self.mx, self.worst = m, (idx[0] + offset,) + tuple(idx[1:])
        self.total += float(d.sum())
        self.n += d.size

    def check(self):
        mean = self.total / max(self.n, 1)
        assert self.mx <= OUT_MAX_ABS and mean <= OUT_MEAN_ABS, (
            f"{self.what}: max |d| = {self.mx:.3e} (<= {OUT_MAX_ABS}) at {self.worst}, mean |d| = {mean:.3e} "
            f"(<= {OUT_MEAN_ABS}) over {self.n} values")
        return self.mx, mean


def assert_lse_close(got: np.ndarray, want: np.ndarray):
    d = np.abs(got - want)
    assert float(d.max()) <= LSE_MAX_ABS, f"lse: max |d| = {float(d.max()):.3e}"


def assert_selection_equal(got: np.ndarray, want: np.ndarray, rows=None):
    if not np.array_equal(got, want):
        bad = np.argwhere((got != want).any(axis=-1))
        r, i = bad[0][0], bad[0][1]
        row = rows[i] if rows is not None else i
        raise AssertionError(f"selection differs at {len(bad)} (group,row) pairs; first group {r} row {row}: "
                             f"got {got[r, i].tolist()} want {want[r, i].tolist()}")


def check_kv2q(kv, sel_oracle: np.ndarray, oracle_mod, B_k: int = 128):
    """CSR offsets/entries equal the oracle's inversion; the work list covers every entry once."""
    L = kv.layout
    off_o, ent_o = oracle_mod.kv2q(sel_oracle, B_k)
    off = kv.offsets().cpu().numpy()
    ent = kv.entries().cpu().numpy()
    for r in range(L.H_kv):
        assert np.array_equal(off[r].astype(np.int64), off_o[r]), f"offsets differ for group {r}"
        n = int(off_o[r, -1])
        assert np.array_equal(ent[r, :n], ent_o[r]), f"entries differ for group {r}"
    wi = kv.window_items().cpu().numpy()
    n_items = int(wi[-1])
    assert n_items <= L.max_items
    items = kv.items(n_items).cpu().numpy() if n_items else np.zeros((0, 4), np.int32)
    covered = [np.zeros(int(off_o[r, -1]), dtype=np.int32) for r in range(L.H_kv)]
    for w in range(L.n_windows):
        for it in items[wi[w]:wi[w + 1]]:
            r, b, start, ln = (int(x) for x in it)
            assert 1 <= ln <= L.chunk
            assert off_o[r, b] <= start and start + ln <= off_o[r, b + 1], "item outside its block's list"
            rows = ent_o[r][start:start + ln] // L.k
            assert rows.min() >= w * L.window and rows.max() < (w + 1) * L.window, "item outside its window"
            covered[r][start:start + ln] += 1
    for r in range(L.H_kv):
        assert (covered[r] == 1).all(), f"work list does not cover group {r}'s entries exactly once"
    return n_items
