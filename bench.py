#!/usr/bin/env python
"""Benchmark of the B200 MSA forward hot path (one JSON line on rank 0).

A step is one pass of the whole hot path over one batch of synthetic input: the 128K-token planted
prefill (index Top-k -> KV->Q inversion -> KV-outer attention -> LSE combine) followed by one decode
step of 64 sequences against 16K-128K token caches. `value` is prefill tokens/s over all ranks
(each rank processes its own independent sequence: weak scaling, no collective on the data path);
decode tokens/s and every kernel's roofline fraction are reported alongside.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {msa,reference}]

--impl reference times the plain CPU oracle (the reference arm of this build) on the host cores,
on a bounded sample of the same workload, and prints the same metric.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_long_idx_b200 import replicas, roofline, synth  # noqa: E402

METRIC = "MSA prefill tokens/s @N=128K (64q/4kv heads), decode tok/s; % of roofline"
UNIT = "tokens/s"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["msa", "reference"], default="msa")
    ap.add_argument("--workload", default=synth.P128K.name, choices=sorted(synth.PREFILL_CONFIGS))
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-varlen", action="store_true", help="skip the packed-batch (varlen) prefill leg")
    ap.add_argument("--no-backward", action="store_true", help="skip the main-branch backward leg")
    ap.add_argument("--no-long", action="store_true", help="skip the 1M-token prefill leg")
    ap.add_argument("--no-fp8", action="store_true", help="skip the FP8 main-branch leg")
    ap.add_argument("--decode-workload", default=synth.DECODE64.name, choices=sorted(synth.DECODE_CONFIGS))
    ap.add_argument("--e2e-steps", type=int, default=8,
                    help="pipelined host-buffer steps (the first input copy and the last output copy are not overlapped)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="target CPU-oracle sample time")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--rows-per-pass", type=int, default=0, help="cap the prefill partial buffer (0 = whole N)")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one ncu capture of a smaller case of
# the same kernel, per query row of the launch; partial outputs grow in proportion to the rows, so a
# full launch is the per-row figure times its rows. A figure only applies to the kernel source it was
# measured on (the kernel's own .cu file, by hash): after any change to it the bench reports null.
PROFILED_TRAFFIC = {
    "attn": {"files": ("sparse_attn.cu",), "sha256_16": "b3f4e84dc09c6d39",
             "bytes_per_row": (379.072e6 + 2.124692e9) / 8192,
             "capture": "ncu capture of sparse_attn_kernel<128, 16, 0> on the N=32768 prefill, one 8192-row pass"},
    "attn_fp8": {"files": ("sparse_attn.cu",), "sha256_16": "b3f4e84dc09c6d39",
                 "bytes_per_row": (228.76288e6 + 2.123282e9) / 8192,
                 "capture": "ncu capture of sparse_attn_kernel<128, 16, 1> on the N=32768 prefill, one 8192-row pass"},
    "combine": {"files": ("combine.cu",), "sha256_16": "c171e6105a4b5769",
                "bytes_per_row": (2.181085e9 + 132.157184e6) / 8192,
                "capture": "ncu capture of combine_kernel on the N=32768 prefill, one 8192-row pass"},
}


def profiled_traffic(name, rows_per_launch):
    t = PROFILED_TRAFFIC.get(name)
    if t is None:
        return None
    import hashlib

    m = hashlib.sha256()
    for f in t["files"]:
        with open(os.path.join(ROOT, "block_sparse_long_idx_b200", "csrc", f), "rb") as fh:
            m.update(fh.read())
    if m.hexdigest()[:16] != t["sha256_16"]:
        return None
    return t["bytes_per_row"] * rows_per_launch


# ------------------------------------------------------------------------------------ CPU oracle
def oracle_rate(prefill_inputs, cfg, target_s: float):
    """Oracle rows/s on a bounded sample of the workload's rows (selection + attention, all heads)."""
    import oracle

    o = oracle.default()

    def run(n, seed):
        rows = synth.sample_rows(cfg.N, cfg.B_k, n, seed)
        t0 = time.perf_counter()
        o.prefill_rows(prefill_inputs, rows, cfg.B_k, cfg.k)
        return len(rows), time.perf_counter() - t0

    n0, t0 = run(8, 101)
    n = max(8, int(n0 * target_s / max(t0, 1e-3)))
    n1, t1 = run(n, 202)
    return {"value": n1 / t1, "unit": UNIT, "cores": o.max_threads(), "kind": "oracle",
            "sample": f"{n1} uniformly sampled query rows (plus rows 0, B_k-1, B_k, N-1) of {cfg.name}: "
                      f"index selection + exact sparse attention for all {cfg.H_q} heads, fp64, "
                      f"{t1:.1f} s; value = rows/s"}


def reference_arm(args, rank):
    if rank != 0:
        return
    cfg = synth.PREFILL_CONFIGS[args.workload]
    inputs = synth.prefill_inputs(cfg)
    import oracle

    o = oracle.default()
    per_step = max(args.cpu_seconds / max(args.steps, 1), 2.0)
    times, rows_done = [], []
    for s in range(args.warmup + args.steps):
        rows = synth.sample_rows(cfg.N, cfg.B_k, max(4, int(4 * per_step)), 1000 + s)
        t0 = time.perf_counter()
        o.prefill_rows(inputs, rows, cfg.B_k, cfg.k)
        dt = time.perf_counter() - t0
        if s >= args.warmup:
            times.append(dt)
            rows_done.append(len(rows))
    value = sum(rows_done) / sum(times)
    dec = None
    if not args.no_decode:
        # decode: the first sequences of the decode workload (the same caches the GPU arm builds), timed
        # as one oracle decode call per step
        dfull = synth.DECODE_CONFIGS[args.decode_workload]
        dcfg = dfull.with_(B=4)
        dinp = synth.decode_inputs(dcfg, lens=synth.decode_lens(dfull)[: dcfg.B])
        dts = []
        for s in range(1 + args.steps):
            t0 = time.perf_counter()
            o.decode(dinp, dcfg.B_k, dcfg.k)
            if s >= 1:
                dts.append(time.perf_counter() - t0)
        dec = {"value": dcfg.B * len(dts) / sum(dts), "unit": "tokens/s", "ms_per_step": 1000 * statistics.mean(dts),
               "sample": f"{dcfg.B} sequences of {dfull.name} (cache lengths {dinp['lens'].tolist()}), "
                         "one decode token each: block pooling, Top-k and sparse attention, fp64"}
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * statistics.mean(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": dict(workload_config(cfg, None if args.no_decode else synth.DECODE_CONFIGS[args.decode_workload]),
                           parallelism=f"replicas x{args.gpus} (independent sequences)"),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": o.max_threads(), "kind": "oracle",
                             "sample": f"per step {rows_done[0]} sampled query rows of {cfg.name} "
                                       "(selection + attention, all heads)"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    if dec is not None:
        line["decode"] = dec
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------ GPU arm
def workload_config(cfg, dcfg):
    c = {"workload": cfg.name + (f" + {dcfg.name}" if dcfg else ""), "N": cfg.N, "H_q": cfg.H_q, "H_kv": cfg.H_kv,
         "d_h": cfg.d_h, "d_idx": cfg.d_idx, "B_k": cfg.B_k, "k": cfg.k, "planted": cfg.planted,
         "l2": "flushed before every timed step (512 MB write)"}
    if dcfg:
        c["decode"] = {"B": dcfg.B, "L_max": dcfg.L_max, "lens": f"uniform [{dcfg.len_lo}, {dcfg.len_hi}]"}
    return c


class ClockSampler:
    """Samples SM clock, power and clock-event reasons during the timed region: NVML every 10 ms
    (read-only queries), or `nvidia-smi -lms 50` when the NVML bindings are missing."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown", 0x4: "sw_power_cap"}

    def __init__(self, uuid: str):
        self.uuid = uuid
        self.samples = []  # (sm_mhz, max_mhz, reason bits)
        self.stop = threading.Event()
        self.proc = None
        self.t = None

    def __enter__(self):
        try:
            import pynvml

            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByUUID(self.uuid)
            mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)

            def poll():
                while not self.stop.is_set():
                    try:
                        sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                        rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.samples.append((float(sm), float(mx), int(rs)))
                    except pynvml.NVMLError:
                        pass
                    self.stop.wait(0.01)

            self.t = threading.Thread(target=poll, daemon=True)
            self.t.start()
            return self
        except Exception:  # no NVML bindings: fall back to nvidia-smi
            pass
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.uuid, f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read_smi, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read_smi(self):
        bits = [0x8, 0x40, 0x20, 0x4]
        for line in self.proc.stdout:
            f = [x.strip() for x in line.strip().split(",")]
            if len(f) < 9:
                continue
            try:
                rs = sum(b for b, v in zip(bits, f[5:9]) if v.lower() == "active")
                self.samples.append((float(f[1]), float(f[2]), rs))
            except ValueError:
                continue

    def __exit__(self, *exc):
        self.stop.set()
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.t:
            self.t.join(timeout=5)
        return False

    def summary(self):
        sm = [x[0] for x in self.samples]
        reasons = sorted({nm for _, _, rs in self.samples for b, nm in self.REASONS.items() if rs & b})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_min_mhz": min(sm) if sm else None,
                "sm_max_mhz": self.samples[-1][1] if self.samples else None, "reasons": reasons,
                "samples": len(sm), "source": "nvml" if self.proc is None else "nvidia-smi"}


def kernel_stats(kern, steps, cfg, peaks, dec_bytes=None):
    """Per-kernel time per step and roofline fraction from the traced CUDA-event durations:
    achieved = algorithmic FLOPs or bytes of the kernel per step / its time per step."""
    N, H_q, H_kv, d_h, d_idx, k, B_k = cfg.N, cfg.H_q, cfg.H_kv, cfg.d_h, cfg.d_idx, cfg.k, cfg.B_k
    algo = {"index_topk": ("tensor", roofline.index_branch_flops(N, H_kv, d_idx)),
            "attn": ("tensor", roofline.main_branch_flops(N, H_q, d_h, k, B_k)),
            "combine": ("hbm", roofline.combine_bytes(N, H_q, H_kv, d_h, k, B_k)),
            "kv2q": ("hbm", roofline.kv2q_bytes(N, H_kv, k, B_k))}
    if dec_bytes:
        algo["dec_pool"] = ("hbm", dec_bytes["dec_pool"])
        algo["dec_attn"] = ("hbm", dec_bytes["dec_attn"])
    kstats = {}
    for name, durs in kern.items():
        per_step = sum(durs) / steps
        ent = {"ms_per_step": per_step, "launches_per_step": len(durs) / steps}
        if name in algo:
            bound, work = algo[name]
            if bound == "tensor":
                ach = work / (per_step / 1000.0) / 1e12
                ent.update({"bound": "tensor", "achieved": ach, "unit": "TFLOP/s", "peak": peaks["bf16_tflops"],
                            "frac": ach / peaks["bf16_tflops"], "algorithmic": work})
            else:
                ach = work / (per_step / 1000.0) / 1e9
                ent.update({"bound": "hbm", "achieved": ach, "unit": "GB/s", "peak": peaks["hbm_gbs"],
                            "frac": ach / peaks["hbm_gbs"], "algorithmic": work})
        if name in ("attn", "combine"):
            rows = N / max(1.0, ent["launches_per_step"])
            tr = profiled_traffic(name, rows)
            ent["traffic"] = tr
            if tr is not None:
                ent["traffic_source"] = PROFILED_TRAFFIC[name]["capture"] + ", scaled by rows per launch"
        kstats[name] = ent
    return kstats


def long_prefill_leg(args, rank, world, dev, peaks, flush):
    """Prefill of one 1M-token sequence (8192 KV blocks; i.i.d. inputs as at 32K) in passes of 131072
    query rows: the long-context regime where the index branch's quadratic term dominates."""
    import torch

    import block_sparse_long_idx_b200 as msa

    cfg = synth.P1M.with_(seed=replicas.replica_seed(synth.P1M.seed, rank))
    host = synth.prefill_inputs(cfg)
    t = {n: torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).to(dev) for n, a in host.items()}
    del host
    N, H_q, H_kv, d_h, k = cfg.N, cfg.H_q, cfg.H_kv, cfg.d_h, cfg.k
    rows_pass = 131072
    block_idx = torch.empty((H_kv, N, k), dtype=torch.int32, device=dev)
    L = msa.msa_kv2q_layout_get(N, H_kv, cfg.B_k, k)
    kv = msa.KV2Q(L, torch.empty(L.total_bytes, dtype=torch.uint8, device=dev))
    ws_kv = torch.empty(msa.api.lib.msa_build_kv2q_workspace_size(msa.api.ctypes.byref(L)), dtype=torch.uint8,
                        device=dev)
    ws_pf = torch.empty(msa.msa_sparse_prefill_workspace_size(N, H_q, H_kv, d_h, cfg.B_k, k, rows_pass),
                        dtype=torch.uint8, device=dev)
    ws_idx = torch.empty(256, dtype=torch.uint8, device=dev)
    out = torch.empty_like(t["q"])
    lse = torch.empty((N, H_q), dtype=torch.float32, device=dev)

    def step():
        cur = torch.cuda.current_stream()
        msa.msa_index_topk(t["q_idx"], t["k_idx"], cfg.B_k, k, block_idx=block_idx, workspace=ws_idx, stream=cur)
        msa.api._check("msa_build_kv2q", msa.api.lib.msa_build_kv2q(
            block_idx.data_ptr(), msa.api.ctypes.byref(L), kv.buf.data_ptr(), ws_kv.data_ptr(), ws_kv.numel(),
            cur.cuda_stream))
        msa.msa_sparse_prefill(t["q"], t["k"], t["v"], block_idx, kv, out=out, lse=lse, workspace=ws_pf, stream=cur)

    steps = max(1, min(args.steps, 3))
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    for ws in (ws_idx, ws_kv, ws_pf):
        if msa.msa_get_device_error(ws) != 0:
            raise RuntimeError("device error in the 1M prefill warm-up")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    trace = msa.KernelTrace(64 * steps)
    with trace:
        for st in range(steps):
            flush.zero_()
            ev[st][0].record()
            step()
            ev[st][1].record()
    torch.cuda.synchronize()
    (ms,) = replicas.max_over_ranks([sum(a.elapsed_time(b) for a, b in ev)], device=dev)
    res = {"workload": cfg.name, "value": replicas.aggregate_rate(N * steps, world, ms / 1000.0), "unit": UNIT,
           "ms_per_step": ms / steps, "steps": steps, "rows_per_pass": rows_pass,
           "kernels": kernel_stats(trace.durations(), steps, cfg, peaks),
           "note": "one 1048576-token sequence, i.i.d. inputs; index Top-k, inversion, and attention + combine "
                   "in passes of 131072 query rows; L2 flushed before each step"}
    del t, block_idx, kv, ws_kv, ws_pf, ws_idx, out, lse
    torch.cuda.empty_cache()
    return res


def gpu_arm(args, rank, world):
    import torch
    import torch.distributed as dist

    import block_sparse_long_idx_b200 as msa

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    peaks = load_peaks()
    cfg = synth.PREFILL_CONFIGS[args.workload]
    cfg = cfg.with_(seed=replicas.replica_seed(cfg.seed, rank))  # independent sequence per rank
    dbase = synth.DECODE_CONFIGS[args.decode_workload]
    dcfg = None if args.no_decode else dbase.with_(seed=replicas.replica_seed(dbase.seed, rank))

    host = synth.prefill_inputs(cfg)
    cpu_base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu_base = oracle_rate(host, cfg, args.cpu_seconds)  # before any GPU work

    def to_dev(a):
        return torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).to(dev)

    t = {n: to_dev(a) for n, a in host.items()}
    N, H_q, H_kv, d_h, d_idx, k = cfg.N, cfg.H_q, cfg.H_kv, cfg.d_h, cfg.d_idx, cfg.k
    block_idx = torch.empty((H_kv, N, k), dtype=torch.int32, device=dev)
    L = msa.msa_kv2q_layout_get(N, H_kv, cfg.B_k, k)
    kv = msa.KV2Q(L, torch.empty(L.total_bytes, dtype=torch.uint8, device=dev))
    ws_kv = torch.empty(msa.api.lib.msa_build_kv2q_workspace_size(msa.api.ctypes.byref(L)), dtype=torch.uint8,
                        device=dev)
    ws_pf = torch.empty(msa.msa_sparse_prefill_workspace_size(N, H_q, H_kv, d_h, cfg.B_k, k, args.rows_per_pass),
                        dtype=torch.uint8, device=dev)
    out = torch.empty_like(t["q"])
    lse = torch.empty((N, H_q), dtype=torch.float32, device=dev)
    ws_idx = torch.empty(256, dtype=torch.uint8, device=dev)

    if dcfg:
        dh = synth.decode_inputs(dcfg)
        dt = {n: to_dev(a) for n, a in dh.items()}
        dout = torch.empty_like(dt["q"])
        dlse = torch.empty((dcfg.B, dcfg.H_q), dtype=torch.float32, device=dev)
        dbi = torch.empty((dcfg.B, dcfg.H_kv, dcfg.k), dtype=torch.int32, device=dev)
        ws_dec = torch.empty(msa.api.lib.msa_sparse_decode_workspace_size(
            dcfg.B, dcfg.L_max, dcfg.H_q, dcfg.H_kv, dcfg.d_h, dcfg.d_idx, dcfg.B_k, dcfg.k), dtype=torch.uint8,
            device=dev)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def prefill(inp=None, dst=None):
        inp = t if inp is None else inp
        dst = out if dst is None else dst
        cur = torch.cuda.current_stream()
        msa.msa_index_topk(inp["q_idx"], inp["k_idx"], cfg.B_k, k, block_idx=block_idx, workspace=ws_idx, stream=cur)
        msa.api._check("msa_build_kv2q", msa.api.lib.msa_build_kv2q(
            block_idx.data_ptr(), msa.api.ctypes.byref(L), kv.buf.data_ptr(), ws_kv.data_ptr(), ws_kv.numel(),
            cur.cuda_stream))
        msa.msa_sparse_prefill(inp["q"], inp["k"], inp["v"], block_idx, kv, out=dst, lse=lse, workspace=ws_pf,
                               stream=cur)

    def decode():
        msa.msa_sparse_decode(dt["q"], dt["q_idx"], dt["k_cache"], dt["v_cache"], dt["k_idx_cache"], dt["lens"],
                              dcfg.B_k, dcfg.k, out=dout, lse=dlse, block_idx_out=dbi, workspace=ws_dec)

    for _ in range(args.warmup):
        prefill()
        if dcfg:
            decode()
    torch.cuda.synchronize()
    for ws in (ws_idx, ws_kv, ws_pf) + ((ws_dec,) if dcfg else ()):
        st = msa.msa_get_device_error(ws)
        if st != 0:
            raise RuntimeError(f"device error {msa.status_string(st)} during warm-up")

    uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    trace = msa.KernelTrace(64 * args.steps)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = msa.msa_launch_count()
    with ClockSampler(uuid) as clocks:
        wall0 = time.perf_counter()
        with trace:
            for s in range(args.steps):
                flush.zero_()  # evict L2 between steps (outside the timed events)
                ev[s][0].record()
                prefill()
                ev[s][1].record()
                if dcfg:
                    decode()
                ev[s][2].record()
        torch.cuda.synchronize()
        wall = time.perf_counter() - wall0
    launches = msa.msa_launch_count() - launches0
    if world > 1:
        dist.barrier()
    pf_ms = [e[0].elapsed_time(e[1]) for e in ev]
    dec_ms = [e[1].elapsed_time(e[2]) for e in ev]
    kern = trace.durations()

    pf_total, dec_total = replicas.max_over_ranks([sum(pf_ms), sum(dec_ms)], device=dev)

    # the decode step captured once in a CUDA graph and replayed (how a serving loop would run it)
    decode_graph = None
    if dcfg:
        cs = torch.cuda.Stream()
        cs.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(cs):
            decode()
        torch.cuda.current_stream().wait_stream(cs)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            decode()
        for _ in range(args.warmup):
            graph.replay()
        gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for st in range(args.steps):
            flush.zero_()
            gev[st][0].record()
            graph.replay()
            gev[st][1].record()
        torch.cuda.synchronize()
        (g_ms,) = replicas.max_over_ranks([sum(a.elapsed_time(b) for a, b in gev)], device=dev)
        decode_graph = {"value": world * dcfg.B * args.steps / (g_ms / 1000.0), "unit": UNIT,
                        "ms_per_step": g_ms / args.steps,
                        "note": "the same decode step captured in a CUDA graph and replayed, L2 flushed before each"}
        del graph

    # packed-batch (varlen) prefill of the same model shape: 16 sequences, 131072 tokens in total
    varlen = None
    if not args.no_varlen:
        vcfg = dataclasses.replace(synth.VARLEN128K, seed=replicas.replica_seed(synth.VARLEN128K.seed, rank))
        vin = synth.varlen_inputs(vcfg)
        vt = {n: to_dev(vin[n]) for n in ("q", "k", "v", "q_idx", "k_idx")}
        v_out = torch.empty_like(vt["q"])
        v_lse = torch.empty((vcfg.T, vcfg.H_q), dtype=torch.float32, device=dev)
        v_bi = torch.empty((vcfg.H_kv, vcfg.T, vcfg.k), dtype=torch.int32, device=dev)
        cu_p = vin["cu_seqlens"].ctypes.data_as(msa.api.ctypes.c_void_p)
        v_ws = torch.empty(msa.api.lib.msa_sparse_prefill_varlen_workspace_size(
            cu_p, None, len(vcfg.lens), vcfg.H_q, vcfg.H_kv, vcfg.d_h, vcfg.B_k, vcfg.k, 0), dtype=torch.uint8,
            device=dev)

        def varlen_step():
            msa.msa_sparse_prefill_varlen(vt["q"], vt["k"], vt["v"], vt["q_idx"], vt["k_idx"], vin["cu_seqlens"],
                                          vcfg.B_k, vcfg.k, block_idx=v_bi, out=v_out, lse=v_lse, workspace=v_ws)

        for _ in range(args.warmup):
            varlen_step()
        torch.cuda.synchronize()
        if msa.msa_get_device_error(v_ws) != 0:
            raise RuntimeError("device error in the varlen warm-up")
        vev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for st in range(args.steps):
            flush.zero_()
            vev[st][0].record()
            varlen_step()
            vev[st][1].record()
        torch.cuda.synchronize()
        (vt_ms,) = replicas.max_over_ranks([sum(a.elapsed_time(b) for a, b in vev)], device=dev)
        varlen = {"value": replicas.aggregate_rate(vcfg.T * args.steps, world, vt_ms / 1000.0), "unit": UNIT,
                  "ms_per_step": vt_ms / args.steps, "workload": vcfg.name, "n_seq": len(vcfg.lens),
                  "lens": f"{min(vcfg.lens)}..{max(vcfg.lens)} (seeded mix)",
                  "note": "msa_sparse_prefill_varlen: index branch, inversion, attention and combine in one call"}
        del vt, v_out, v_lse, v_bi, v_ws

    # FP8 main branch on the same workload and selections: E4M3 quantisation of q, k, v (timed, part of
    # the step) and the attention on FP8 tensor cores + combine; index branch and inversion as above
    fp8 = None
    if not args.no_fp8 and d_h == 128:
        f_out = torch.empty_like(out)
        f_lse = torch.empty_like(lse)

        def fp8_step():
            qq, kq, vq = (msa.msa_quantize_e4m3(t[n]) for n in ("q", "k", "v"))
            msa.msa_sparse_prefill_fp8(qq, kq, vq, block_idx, kv, out=f_out, lse=f_lse, workspace=ws_pf)

        for _ in range(args.warmup):
            fp8_step()
        torch.cuda.synchronize()
        if msa.msa_get_device_error(ws_pf) != 0:
            raise RuntimeError("device error in the FP8 warm-up")
        fev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        ftrace = msa.KernelTrace(16 * args.steps)
        with ftrace:
            for st in range(args.steps):
                flush.zero_()
                fev[st][0].record()
                fp8_step()
                fev[st][1].record()
        torch.cuda.synchronize()
        (f_ms,) = replicas.max_over_ranks([sum(a.elapsed_time(b) for a, b in fev)], device=dev)
        fk = {n: sum(d) / args.steps for n, d in ftrace.durations().items()}
        peak8 = 2.0 * peaks["bf16_tflops"]
        ach8 = roofline.main_branch_flops(N, H_q, d_h, k, cfg.B_k) / (fk["attn"] / 1000.0) / 1e12
        qb = (roofline.quant_bytes(N, H_q, d_h) + 2 * roofline.quant_bytes(N, H_kv, d_h))
        fp8 = {"ms_per_step": f_ms / args.steps, "kernels_ms": fk,
               "roofline": {"kernel": "attn (fp8)", "bound": "tensor", "achieved": ach8, "unit": "TFLOP/s",
                            "peak": peak8, "frac": ach8 / peak8,
                            "peak_source": "measured bf16 burst x 2 (nominal FP8 / bf16 dense ratio)",
                            "traffic": profiled_traffic("attn_fp8", N), "traffic_source":
                                PROFILED_TRAFFIC["attn_fp8"]["capture"] + ", scaled by rows per launch"},
               "quant": {"achieved": qb / (fk["quant"] / 1000.0) / 1e9, "unit": "GB/s", "peak": peaks["hbm_gbs"],
                         "frac": qb / (fk["quant"] / 1000.0) / 1e9 / peaks["hbm_gbs"], "algorithmic": qb},
               "prefill_tokens_per_s": replicas.aggregate_rate(
                   N * args.steps, world,
                   (f_ms + sum(sum(kern.get(n, [0.0])) for n in ("index_topk", "kv2q"))) / 1000.0),
               "note": "E4M3 quantisation of q, k, v + FP8 attention + combine per step; prefill_tokens_per_s "
                       "adds the bf16 index branch and inversion times of the main leg"}
        del f_out, f_lse

    # main-branch backward on the same workload, selections held fixed: gradients of sum(dout * out) in
    # q, k, v from the forward's out and lse of the timed steps
    backward = None
    if not args.no_backward:
        bdout = to_dev(synth.normal_bf16((N, H_q, d_h), cfg.seed, "dout"))
        bdq, bdk, bdv = torch.empty_like(t["q"]), torch.empty_like(t["k"]), torch.empty_like(t["v"])
        b_ws = torch.empty(msa.api.lib.msa_sparse_backward_workspace_size(N, H_q, H_kv, d_h, cfg.B_k, k, d_idx, 0),
                           dtype=torch.uint8, device=dev)

        def backward_step(with_kl):
            kw = dict(q_idx=t["q_idx"], k_idx=t["k_idx"], kl_weight=1.0 / (N * H_kv)) if with_kl else {}
            msa.msa_sparse_backward(t["q"], t["k"], t["v"], out, lse, bdout, block_idx, kv, cfg.B_k, k, dq=bdq,
                                    dk=bdk, dv=bdv, workspace=b_ws, **kw)

        def timed_backward(with_kl):
            for _ in range(args.warmup):
                backward_step(with_kl)
            torch.cuda.synchronize()
            if msa.msa_get_device_error(b_ws) != 0:
                raise RuntimeError("device error in the backward warm-up")
            bev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)]
            btrace = msa.KernelTrace(16 * args.steps)
            with btrace:
                for st in range(args.steps):
                    flush.zero_()
                    bev[st][0].record()
                    backward_step(with_kl)
                    bev[st][1].record()
            torch.cuda.synchronize()
            (ms,) = replicas.max_over_ranks([sum(a.elapsed_time(b) for a, b in bev)], device=dev)
            return ms, {n: sum(d) / args.steps for n, d in btrace.durations().items()}

        bt_ms, bk = timed_backward(False)
        kl_ms, kl_k = timed_backward(True)
        fl_bwd = roofline.main_branch_backward_flops(N, H_q, d_h, k, cfg.B_k)
        ach = fl_bwd / (bk["bwd_attn"] / 1000.0) / 1e12
        backward = {"value": replicas.aggregate_rate(N * args.steps, world, bt_ms / 1000.0), "unit": UNIT,
                    "ms_per_step": bt_ms / args.steps, "kernels_ms": bk,
                    "roofline": {"kernel": "bwd_attn", "bound": "tensor", "achieved": ach, "unit": "TFLOP/s",
                                 "peak": peaks["bf16_tflops"], "frac": ach / peaks["bf16_tflops"],
                                 "algorithmic": fl_bwd},
                    "with_kl": {"ms_per_step": kl_ms / args.steps, "kernels_ms": kl_k,
                                "note": "the same call also computing the index branch's KL alignment "
                                        "(per-row KL, dq_idx, dk_idx) in the same pass"},
                    "note": "msa_sparse_backward (dq, dk, dv; selections fixed), first path on mma.sync"}
        del bdout, bdq, bdk, bdv, b_ws

    # end-to-end through the public API with host buffers (pinned), copies inside the timed region:
    # every step copies its inputs in and its output back; device inputs and outputs are double
    # buffered so step s+1's inputs stream in and step s-1's output streams out while step s computes
    e2e = None
    if args.e2e_steps > 0:
        pin = {n: torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).pin_memory()
               for n, a in host.items()}
        out_h = [torch.empty(out.shape, dtype=out.dtype, pin_memory=True) for _ in range(2)]
        h2d = sum(p.numel() * p.element_size() for p in pin.values())
        d2h = out_h[0].numel() * out_h[0].element_size()
        dev_in = [t, {n: torch.empty_like(x) for n, x in t.items()}]
        dev_out = [out, torch.empty_like(out)]
        s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        in_ready = [torch.cuda.Event() for _ in range(args.e2e_steps)]
        comp_done = [torch.cuda.Event() for _ in range(args.e2e_steps)]
        out_done = [torch.cuda.Event() for _ in range(args.e2e_steps)]
        flush.zero_()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        s_comp.wait_event(e0)
        s_out.wait_event(e0)
        for st in range(args.e2e_steps):
            bsel = st & 1
            with torch.cuda.stream(s_in):
                if st >= 2:
                    s_in.wait_event(comp_done[st - 2])  # step st-2 has finished reading these inputs
                for n in t:
                    dev_in[bsel][n].copy_(pin[n], non_blocking=True)
                in_ready[st].record(s_in)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(in_ready[st])
                if st >= 2:
                    s_comp.wait_event(out_done[st - 2])  # step st-2's output has been copied out
                prefill(dev_in[bsel], dev_out[bsel])
                comp_done[st].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[st])
                out_h[bsel].copy_(dev_out[bsel], non_blocking=True)
                out_done[st].record(s_out)
        s_in.wait_stream(s_out)
        s_in.wait_stream(s_comp)
        e1.record(s_in)
        torch.cuda.synchronize()
        (te,) = replicas.max_over_ranks([e0.elapsed_time(e1)], device=dev)
        e2e = {"value": replicas.aggregate_rate(N * args.e2e_steps, world, te / 1000.0), "unit": UNIT,
               "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h,
               "steps": args.e2e_steps,
               "note": "prefill through the public API on host buffers: every step copies its inputs in from "
                       "pinned memory and its output back; inputs/outputs double-buffered on the device so the "
                       "copies of neighbouring steps overlap the current step's kernels"}

    # 1M-token prefill (passes of 131072 rows): release the 128K workload's large buffers first
    long_prefill = None
    if not args.no_long:
        ws_pf = dt = dev_in = dev_out = pin = out_h = None  # noqa: F841 (drop the 128K buffers)
        torch.cuda.empty_cache()
        long_prefill = long_prefill_leg(args, rank, world, dev, peaks, flush)

    if rank != 0:
        return
    value = replicas.aggregate_rate(N * args.steps, world, pf_total / 1000.0)
    dec_bytes = (roofline.decode_bytes(dh["lens"], dcfg.H_q, dcfg.H_kv, dcfg.d_h, dcfg.d_idx, dcfg.k, dcfg.B_k)
                 if dcfg else None)
    kstats = kernel_stats(kern, args.steps, cfg, peaks, dec_bytes)
    # dominant kernel of the prefill step
    dom = max((n for n in ("index_topk", "attn", "combine") if n in kstats), key=lambda n: kstats[n]["ms_per_step"])
    d = kstats[dom]
    roof = {"kernel": dom, "bound": d["bound"], "achieved": d["achieved"], "peak": d["peak"], "unit": d["unit"],
            "frac": d["frac"], "traffic": d.get("traffic"), "peak_source": peaks["source"] + " (burst)"}
    if d.get("traffic") is not None:
        roof["traffic_source"] = d["traffic_source"]
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": (pf_total + dec_total) / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(workload_config(cfg, dcfg), parallelism=f"replicas x{world} (independent sequences)"),
            "prefill_ms_per_step": pf_total / args.steps,
            "decode": ({"value": world * dcfg.B * args.steps / (dec_total / 1000.0), "unit": UNIT,
                        "ms_per_step": dec_total / args.steps} if dcfg else None),
            "decode_graph": decode_graph,
            "roofline": roof, "kernels": kstats, "cpu_baseline": cpu_base, "e2e": e2e, "varlen": varlen,
            "backward": backward, "long_prefill": long_prefill, "fp8": fp8,
            "gpu_launches": int(launches), "clocks": clocks.summary(), "wall_s_timed": wall}
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    rank, world, _ = replicas.rank_info()
    if args.impl == "reference":
        reference_arm(args, rank)
        return
    if world > 1:
        replicas.init("nccl", timeout_s=300)
    try:
        gpu_arm(args, rank, world)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
