#!/usr/bin/env python
"""Benchmark of the W4A16 hot path on B200 (one JSON line on stdout).

Headline (the `value`): W4A16 decode GEMV GB/s on the Llama-7B attention
projection workload -- W[4096, 4096] bf16 quantized group-128 asymmetric uint4,
M = 1 bf16 activation.  One step = one decode sweep of 64 GEMV launches over 64
distinct packed copies (557 MB of artifacts, > 4x the 126 MB L2, so every
launch streams its weights from HBM), replayed from a CUDA graph.  Algorithmic
bytes per launch: 0.5 B/weight packed codes + 4 B per group (fp16 scale+zero)
+ 2 B per activation in and output out = 8,929,280 B.

The same line carries the other two metric items (quantize GB/s, GEMM
TFLOP/s) and secondary decode shapes under "secondary", the roofline of the
dominant kernel, an end-to-end number through the C ABI with host buffers,
clocks sampled during the timed regions, and the CPU-oracle baseline.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]

With N > 1 (torchrun) every rank runs an independent replica (the path does
not shard: "replicas only"); timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W4A16 GEMV GB/s & %HBM roofline (4096², g128, M=1); quantize GB/s; GEMM TFLOP/s"
NCOPY = 64
D = 4096
G128 = 128


def gemv_bytes(N: int, K: int, M: int, symmetric: bool, g: int = 128) -> int:
    per_group = 2 if symmetric else 4
    return N * K // 2 + (N * K // g) * per_group + 2 * M * (K + N)


def quant_bytes(N: int, K: int, symmetric: bool, g: int = 128) -> int:
    per_group = 2 if symmetric else 4
    return N * K * 2 + N * K // 2 + (N * K // g) * per_group


def source_digest(files) -> str:
    """sha256 over the CUDA sources a kernel is compiled from; DRAM counters
    taken from an older version of those sources do not apply."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "w4a16_bit_gemm_b200", "csrc")
    for name in sorted(files):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()


def kernel_traffic(name: str):
    """DRAM bytes per launch from a committed ncu summary, or None when it is
    missing or was taken on different kernel sources."""
    path = os.path.join(ROOT, "profiles", name)
    try:
        with open(path) as f:
            rec = json.load(f)
        if rec.get("source_sha256") != source_digest(rec["kernel_sources"]):
            return None
    except (OSError, ValueError, KeyError):
        return None
    return rec.get("dram_bytes_per_launch")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# --------------------------------------------------------------------------
# distributed plumbing (replicas only: a barrier and a max of timings)
# --------------------------------------------------------------------------

class Dist:
    """One process per GPU (RANK / LOCAL_RANK / WORLD_SIZE / MASTER_* from the
    launcher).  The backend is NCCL; WQ_DIST_BACKEND=gloo runs the same
    plumbing on CPU processes (tests)."""

    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.backend = os.environ.get("WQ_DIST_BACKEND", "nccl")
        self.pg = False
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            if self.backend == "nccl":
                torch.cuda.set_device(self.local)
                dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                        device_id=torch.device("cuda", self.local))
            else:
                dist.init_process_group(self.backend, timeout=datetime.timedelta(seconds=120))
            self.pg = True

    def barrier(self):
        if self.pg:
            import torch.distributed as dist
            dist.barrier()

    def max(self, v: float) -> float:
        if not self.pg:
            return v
        import torch.distributed as dist
        t = torch.tensor([v], dtype=torch.float64, device="cuda" if self.backend == "nccl" else "cpu")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            import torch.distributed as dist
            dist.destroy_process_group()


# --------------------------------------------------------------------------
# clocks sampled during the timed regions
# --------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="wq_clocks_", suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        out = {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        if self.proc is None:
            return out
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return out
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for _, _, flags in rows:
            for n, v in zip(names, flags):
                if v.lower().startswith("active"):
                    reasons.add(n)
        out["sm_mhz"] = statistics.median(r[0] for r in rows)
        out["sm_max_mhz"] = max(r[1] for r in rows)
        out["reasons"] = sorted(reasons)
        out["samples"] = len(rows)
        return out


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------

def timed_graph(graph: torch.cuda.CUDAGraph, steps: int, warmup: int, dist: Dist):
    for _ in range(warmup):
        graph.replay()
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        graph.replay()
    e.record()
    torch.cuda.synchronize()
    dist.barrier()
    return s.elapsed_time(e) / 1e3  # seconds


def capture(fn) -> torch.cuda.CUDAGraph:
    fn()  # eager warm-up (first-call set-up happens outside the capture)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def replicate(p, n):
    from w4a16_bit_gemm_b200 import binding as b
    return [b.PackedLinear(p.qweight.clone(), p.scales.clone(), None if p.zeros is None else p.zeros.clone(),
                           p.d_out, p.d_in, p.group_size, p.symmetric) for _ in range(n)]


def gemv_sweep(b, packs, X, Y):
    def fn():
        for i, p in enumerate(packs):
            b.linear_w4a16(X[i], p, out=Y[i])
    return fn


def bench_gemv_shape(b, syn, wl, ci, M, copies, steps, warmup, dist):
    c = wl.cases[ci]
    W = syn.case_weight(wl, ci, "cuda")
    p0 = b.quantize_rtn(W, c.group_size, c.symmetric)
    del W
    packs = replicate(p0, copies)
    X = [syn.case_activations(wl, ci, M, "cuda") for _ in range(1)] * copies
    Y = [torch.empty(M, c.d_out, dtype=torch.bfloat16, device="cuda") for _ in range(copies)]
    g = capture(gemv_sweep(b, packs, X, Y))
    t = dist.max(timed_graph(g, steps, warmup, dist))
    per_launch = t / (steps * copies)
    nbytes = gemv_bytes(c.d_out, c.d_in, M, c.symmetric, c.group_size)
    del g, packs, Y
    torch.cuda.empty_cache()
    return {"shape": f"{c.d_out}x{c.d_in}", "M": M, "symmetric": c.symmetric, "us_per_launch": per_launch * 1e6,
            "GBps": nbytes / per_launch / 1e9, "bytes_per_launch": nbytes}


def bench_whole_model(b, syn, args, dist, hbm):
    """Config 5: quantize the 160 weight matrices of a 32-layer 7B-shaped
    decoder (qkv, o, gate, up, down), report the artifact bytes against
    P*4/8 + scale/zero bytes, then time one M=1 decode sweep over the 160
    layers in model order (one CUDA graph; 3.44 GB of artifacts per sweep, far
    above L2, so every launch streams from HBM)."""
    wl = syn.WHOLE_MODEL
    cases = wl.cases
    Ws = [syn.case_weight(wl, i, "cuda") for i in range(len(cases))]
    packs = [b.quantize_rtn(W, 128, False) for W in Ws]  # allocation + warm-up
    torch.cuda.synchronize()
    P = sum(c.d_out * c.d_in for c in cases)
    art = sum(p.nbytes() for p in packs)
    qbytes = sum(quant_bytes(c.d_out, c.d_in, False) for c in cases)
    dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 3
    e0.record()
    for _ in range(reps):
        for W, p in zip(Ws, packs):
            b.quantize_rtn(W, 128, False, out=p)
    e1.record()
    torch.cuda.synchronize()
    tq = dist.max(e0.elapsed_time(e1) / 1e3) / reps
    del Ws
    torch.cuda.empty_cache()
    X = [syn.case_activations(wl, i, 1, "cuda") for i in range(len(cases))]
    Y = [torch.empty(1, c.d_out, dtype=torch.bfloat16, device="cuda") for c in cases]

    def sweep():
        for i, p in enumerate(packs):
            b.linear_w4a16(X[i], p, out=Y[i])
    g = capture(sweep)
    steps = max(10, min(200, args.steps))
    t = dist.max(timed_graph(g, steps, 3, dist)) / steps
    sweep_bytes = sum(gemv_bytes(c.d_out, c.d_in, 1, False) for c in cases)
    del g, packs, X, Y
    torch.cuda.empty_cache()
    return {"layers": len(cases), "params": P, "artifact_bytes": art,
            "payload_bytes_P_x_4_over_8": P * 4 // 8, "scale_zero_bytes": art - P * 4 // 8,
            "bits_per_weight": 8.0 * art / P,
            "quantize_all_ms": tq * 1e3, "quantize_all_GBps": qbytes / tq / 1e9,
            "gemv_sweep_ms": t * 1e3, "gemv_sweep_bytes": sweep_bytes, "gemv_sweep_GBps": sweep_bytes / t / 1e9,
            "gemv_sweep_frac_of_measured_hbm": sweep_bytes / t / 1e9 / hbm}


def run_ours(args, dist: Dist):
    from w4a16_bit_gemm_b200 import binding as b
    from w4a16_bit_gemm_b200 import synthetic as syn

    hbm, tf_burst, tf_sust, peak_src = load_peaks()
    dev = torch.cuda.current_device()
    sampler = ClockSampler(dev)

    # ---------------- headline: cfg2 GEMV M=1 decode sweep ----------------
    wl = syn.ATTN
    c = wl.cases[0]
    W = syn.case_weight(wl, 0, "cuda")
    p0 = b.quantize_rtn(W, G128, False)
    packs = replicate(p0, NCOPY)
    X_all = syn.activations(NCOPY, D, wl.seed, 77, "cuda", channel_outlier_frac=0.001)
    Y_all = torch.empty(NCOPY, D, dtype=torch.bfloat16, device="cuda")
    Xv = [X_all[i:i + 1] for i in range(NCOPY)]
    Yv = [Y_all[i:i + 1] for i in range(NCOPY)]
    graph = capture(gemv_sweep(b, packs, Xv, Yv))
    st, flags = b.device_error()
    if st != b.WQ_OK:
        raise RuntimeError(f"device status after warm-up: {st} flags {flags}")

    sampler.start()
    t_head = dist.max(timed_graph(graph, args.steps, args.warmup, dist))
    per_launch = t_head / (args.steps * NCOPY)
    bytes_launch = gemv_bytes(D, D, 1, False)
    value = bytes_launch * NCOPY * args.steps * dist.world / t_head / 1e9
    achieved = bytes_launch / per_launch / 1e9

    # ---------------- end to end through the C ABI with host buffers ----------------
    X_host = X_all.cpu().pin_memory()
    Y_host = torch.empty_like(Y_all, device="cpu").pin_memory()
    stream = torch.cuda.current_stream()
    e2e_steps = max(10, min(args.steps, 500))
    for _ in range(3):
        X_all.copy_(X_host, non_blocking=True)
        graph.replay()
        Y_host.copy_(Y_all, non_blocking=True)
        stream.synchronize()
    dist.barrier()
    t0 = time.perf_counter()
    for _ in range(e2e_steps):
        X_all.copy_(X_host, non_blocking=True)
        graph.replay()
        Y_host.copy_(Y_all, non_blocking=True)
        stream.synchronize()
    t_e2e = dist.max(time.perf_counter() - t0)
    dist.barrier()
    e2e_value = bytes_launch * NCOPY * e2e_steps * dist.world / t_e2e / 1e9
    del graph, packs

    # ---------------- secondary: quantize GB/s, dequant GB/s ----------------
    secondary = {}
    QC = 16
    Ws = [W] + [W.clone() for _ in range(QC - 1)]
    qpacks = replicate(p0, QC)

    def qfn():
        for i in range(QC):
            b.quantize_rtn(Ws[i], G128, False, out=qpacks[i])
    gq = capture(qfn)
    qsteps = max(5, args.steps // 20)
    tq = dist.max(timed_graph(gq, qsteps, 3, dist)) / (qsteps * QC)
    qb = quant_bytes(D, D, False)
    secondary["quantize"] = {"shape": "4096x4096", "GBps": qb / tq / 1e9, "us_per_launch": tq * 1e6,
                             "bytes_per_launch": qb, "frac_of_measured_hbm": qb / tq / 1e9 / hbm}
    # quantization with the per-group MSE-optimal clipping search: throughput and
    # the squared reconstruction error relative to RTN on the same weights
    def qcfn():
        for i in range(QC):
            b.quantize_clip_mse(Ws[i], G128, False, out=qpacks[i])
    gqc = capture(qcfn)
    tqc = dist.max(timed_graph(gqc, max(3, qsteps // 4), 3, dist)) / (max(3, qsteps // 4) * QC)
    p_clip = b.quantize_clip_mse(W, G128, False)
    Wd = W.double()
    err_clip = float(((Wd - b.dequantize(p_clip).double()) ** 2).sum())
    err_rtn = float(((Wd - b.dequantize(p0).double()) ** 2).sum())
    secondary["quantize_clip_mse"] = {"shape": "4096x4096", "GBps": qb / tqc / 1e9, "us_per_launch": tqc * 1e6,
                                      "frac_of_measured_hbm": qb / tqc / 1e9 / hbm,
                                      "sq_error_vs_rtn": err_clip / err_rtn}
    del gqc, p_clip, Wd
    # AWQ per-input-channel scaling search (11 alphas) with 512 calibration
    # tokens carrying the 0.1% x50 activation channels; eager launches (the
    # search holds ~70 launches, ~1 ms of device work, so the host keeps ahead)
    T_CAL = 512
    Xc = syn.activations(T_CAL, D, 21, 2, "cuda", channel_outlier_frac=0.001)
    ws = torch.empty(b.wq_awq_workspace_bytes(D, D, T_CAL, G128), dtype=torch.uint8, device="cuda")
    short = args.steps < 20  # the short form (profiling runs) times each search once
    for _ in range(1 if short else 3):
        r_awq = b.awq_search(W, Xc, workspace=ws)
    torch.cuda.synchronize()
    dist.barrier()
    asteps = 1 if short else 5
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    for _ in range(asteps):
        r_awq = b.awq_search(W, Xc, workspace=ws)
    ev1.record()
    torch.cuda.synchronize()
    dist.barrier()
    ta = dist.max(ev0.elapsed_time(ev1) / 1e3) / asteps
    a_best = int(r_awq.best.item())
    a_losses = r_awq.losses.cpu()
    secondary["awq_search"] = {"shape": "4096x4096", "calib_tokens": T_CAL, "alphas": 11,
                               "ms_per_search": ta * 1e3, "alpha": a_best / 10.0,
                               "loss_vs_rtn": float(a_losses[a_best] / a_losses[0])}
    del r_awq, ws
    # GPTQ (fp64 Hessian, inverse factor and error-feedback sweep), the page's
    # setting: symmetric, group 128, act-order; same calibration activations
    gws = torch.empty(b.wq_gptq_workspace_bytes(D, D), dtype=torch.uint8, device="cuda")
    for _ in range(1 if short else 2):
        p_g, _ = b.gptq(W, Xc, G128, True, True, workspace=gws)
    torch.cuda.synchronize()
    dist.barrier()
    gsteps = 1 if short else 3
    ev0.record()
    for _ in range(gsteps):
        p_g, _ = b.gptq(W, Xc, G128, True, True, workspace=gws)
    ev1.record()
    torch.cuda.synchronize()
    dist.barrier()
    tgq = dist.max(ev0.elapsed_time(ev1) / 1e3) / gsteps
    p_r = b.quantize_rtn(W, G128, True)
    Wd64, Xd64 = W.double(), Xc.double()
    e_g = float((((Wd64 - b.dequantize(p_g).double()) @ Xd64.T) ** 2).sum())
    e_r = float((((Wd64 - b.dequantize(p_r).double()) @ Xd64.T) ** 2).sum())
    secondary["gptq"] = {"shape": "4096x4096", "calib_tokens": T_CAL, "symmetric": True, "act_order": True,
                         "ms_per_layer": tgq * 1e3, "output_sq_error_vs_rtn": e_g / e_r}
    del gws, p_g, p_r, Wd64, Xd64, Xc
    What = [torch.empty(D, D, dtype=torch.bfloat16, device="cuda") for _ in range(QC)]

    def dfn():
        for i in range(QC):
            b.dequantize(qpacks[i], out=What[i])
    gd = capture(dfn)
    td = dist.max(timed_graph(gd, qsteps, 3, dist)) / (qsteps * QC)
    secondary["dequantize"] = {"shape": "4096x4096", "GBps": qb / td / 1e9, "us_per_launch": td * 1e6,
                               "frac_of_measured_hbm": qb / td / 1e9 / hbm}
    # references for the same M=1 layer: the pages' path B (full dequantize,
    # then a bf16 matmul) and the unquantized bf16 layer, both through
    # torch.matmul; timed locally (no collective), and an error in a reference
    # leg is reported instead of stopping the benchmark
    try:
        Xr = syn.case_activations(syn.ATTN, 0, 1, "cuda")
        Yr = [torch.empty(1, D, dtype=torch.bfloat16, device="cuda") for _ in range(QC)]

        def path_b():
            for i in range(QC):
                b.dequantize(qpacks[i], out=What[i])
                torch.matmul(Xr, What[i].t(), out=Yr[i])

        def dense():
            for i in range(QC):
                torch.matmul(Xr, Ws[i].t(), out=Yr[i])

        def local_time(graph, reps):
            for _ in range(3):
                graph.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(reps):
                graph.replay()
            e1.record()
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) / 1e3 / (reps * QC)

        t_pb = local_time(capture(path_b), qsteps)
        t_dn = local_time(capture(dense), qsteps)
        secondary["references_m1"] = {
            "shape": "4096x4096", "M": 1, "copies": QC,
            "path_b_dequantize_then_matmul_us": t_pb * 1e6,
            "bf16_matmul_us": t_dn * 1e6,
            "bf16_matmul_GBps": (D * D * 2 + 2 * 2 * D) / t_dn / 1e9,
            "w4a16_gemv_speedup_vs_bf16": t_dn / per_launch,
            "w4a16_gemv_speedup_vs_path_b": t_pb / per_launch}
        del Yr
    except Exception as ex:  # noqa: BLE001
        secondary["references_m1"] = {"error": repr(ex)[:300]}
    del gq, gd, Ws, qpacks, What, W
    torch.cuda.empty_cache()

    # ---------------- secondary decode shapes ----------------
    ssteps = max(5, args.steps // 10)
    secondary["gemv"] = []
    for (wlx, ci, M) in ((syn.ATTN, 0, 8), (syn.MLP, 0, 1), (syn.MLP, 0, 16), (syn.MLP, 2, 1), (syn.MLP, 2, 4)):
        r = bench_gemv_shape(b, syn, wlx, ci, M, 24, ssteps, 3, dist)
        r["frac_of_measured_hbm"] = r["GBps"] / hbm
        secondary["gemv"].append(r)

    # ---------------- W8A16 (symmetric INT8, per-channel) ----------------
    # decode GEMV M=1 and M=16 on the 4096 x 4096 projection, 64 distinct copies
    # per sweep (1.07 GB > L2), then the prefill GEMM at M=2048 on 8192 x 8192
    secondary["w8a16"] = []
    W8 = syn.case_weight(syn.ATTN, 0, "cuda")
    p8 = b.quantize_w8(W8)
    del W8
    p8s = [b.PackedLinearW8(p8.qweight.clone(), p8.scales.clone(), D, D, D) for _ in range(NCOPY)]
    for M in (1, 16):
        X8 = syn.case_activations(syn.ATTN, 0, M, "cuda")
        Y8 = [torch.empty(M, D, dtype=torch.bfloat16, device="cuda") for _ in range(NCOPY)]

        def w8fn():
            for i in range(NCOPY):
                b.linear_w8a16(X8, p8s[i], out=Y8[i])
        g8 = capture(w8fn)
        t8 = dist.max(timed_graph(g8, ssteps, 3, dist)) / (ssteps * NCOPY)
        nb8 = D * D + 2 * D + 2 * M * (D + D)
        secondary["w8a16"].append({"shape": "4096x4096", "M": M, "group": "per-channel", "us_per_launch": t8 * 1e6,
                                   "GBps": nb8 / t8 / 1e9, "bytes_per_launch": nb8,
                                   "frac_of_measured_hbm": nb8 / t8 / 1e9 / hbm})
        del g8, Y8
    del p8s, p8
    torch.cuda.empty_cache()
    cc = syn.PREFILL.cases[0]
    Wg8 = syn.case_weight(syn.PREFILL, 0, "cuda")
    pg8 = b.quantize_w8(Wg8, G128)
    del Wg8
    Xg8 = syn.case_activations(syn.PREFILL, 0, 2048, "cuda")
    Yg8 = torch.empty(2048, cc.d_out, dtype=torch.bfloat16, device="cuda")
    gg8 = capture(lambda: b.linear_w8a16(Xg8, pg8, out=Yg8))
    tg8 = dist.max(timed_graph(gg8, 20, 3, dist)) / 20
    fl8 = 2.0 * 2048 * cc.d_out * cc.d_in
    secondary["w8a16"].append({"shape": f"{cc.d_out}x{cc.d_in}", "M": 2048, "group": 128,
                               "ms_per_launch": tg8 * 1e3, "TFLOPs": fl8 / tg8 / 1e12,
                               "frac_of_measured_bf16": fl8 / tg8 / 1e12 / tf_burst})
    del gg8, pg8, Xg8, Yg8
    torch.cuda.empty_cache()

    # ---------------- GEMM TFLOP/s (config 4) ----------------
    secondary["gemm"] = []
    for (ci, M) in ((0, 512), (0, 2048), (1, 8192)):
        cc = syn.PREFILL.cases[ci]
        Wg = syn.case_weight(syn.PREFILL, ci, "cuda")
        pg = b.quantize_rtn(Wg, G128, False)
        del Wg
        Xg = syn.case_activations(syn.PREFILL, ci, M, "cuda")
        Yg = torch.empty(M, cc.d_out, dtype=torch.bfloat16, device="cuda")
        gg = capture(lambda: b.linear_w4a16(Xg, pg, out=Yg))
        gsteps = max(20, min(50, args.steps // 40))
        tg = dist.max(timed_graph(gg, gsteps, 2, dist)) / gsteps
        flops = 2.0 * M * cc.d_out * cc.d_in
        tfl = flops / tg / 1e12
        secondary["gemm"].append({"M": M, "N": cc.d_out, "K": cc.d_in, "ms_per_launch": tg * 1e3, "TFLOPs": tfl,
                                  "frac_of_measured_bf16_burst": tfl / tf_burst,
                                  "frac_of_measured_bf16_sustained": tfl / tf_sust})
        del gg, pg, Xg, Yg
        torch.cuda.empty_cache()
    # ---------------- config 5: the whole 7B-shaped decoder weight set ----------------
    secondary["whole_model"] = bench_whole_model(b, syn, args, dist, hbm)

    clocks = sampler.stop()
    st, flags = b.device_error()
    if st != b.WQ_OK:
        raise RuntimeError(f"device status after the bench: {st} flags {flags}")

    # the numbers the metric names, last on the line (a stored tail keeps them)
    g_by = {(r["shape"], r["M"]): r for r in secondary["gemv"]}
    secondary["summary"] = {
        "quantize_GBps": secondary["quantize"]["GBps"],
        "dequantize_GBps": secondary["dequantize"]["GBps"],
        "gemm_TFLOPs": {f"{r['M']}x{r['N']}x{r['K']}": r["TFLOPs"] for r in secondary["gemm"]},
        "gemv_GBps": {f"{k[0]} M={k[1]}": v["GBps"] for k, v in g_by.items()},
        "whole_model": {k: secondary["whole_model"][k] for k in ("quantize_all_GBps", "artifact_bytes",
                                                                  "gemv_sweep_GBps", "gemv_sweep_frac_of_measured_hbm")},
    }

    traffic = kernel_traffic("gemv_traffic.json")

    out = {
        "metric": METRIC,
        "value": value,
        "unit": "GB/s",
        "n_gpus": dist.world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": t_head / args.steps * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 activations x uint4 weights, fp32 accumulate",
        "data": "synthetic (seeded N(0,0.02) weights with 0.1% column outliers x20; N(0,1) activations with 0.1% channels x50)",
        "config": {"workload": "llama7b-attn-proj W[4096,4096] g128 asym uint4, W4A16 GEMV M=1",
                   "step": f"{NCOPY} GEMV launches over {NCOPY} distinct packed copies (CUDA graph)",
                   "l2": f"inputs larger than L2: {NCOPY} artifact copies = {NCOPY * p0.nbytes() / 1e6:.0f} MB",
                   "parallelism": f"replicas x{dist.world}"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "traffic": traffic, "peak_source": f"{peak_src} hbm_gbs"},
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": NCOPY * D * 2,
                "d2h_bytes_per_step": NCOPY * D * 2},
        "gpu_launches": args.steps * NCOPY,
        "clocks": clocks,
        "secondary": secondary,
    }
    return out


# --------------------------------------------------------------------------
# CPU oracle (baseline and reference arm)
# --------------------------------------------------------------------------

def oracle_gemv_sample(n_launch: int, nthreads: int | None = None):
    """The oracle as it stands on the same workload: for each launch of the
    sample, unpack the artifact, dequantize and run the fp64 linear layer
    (on every host core unless nthreads is given)."""
    import oracle
    from w4a16_bit_gemm_b200 import synthetic as syn
    W = syn.case_weight(syn.ATTN, 0, "cpu")
    Wb = W.view(torch.int16).numpy().view(np.uint16)
    q, s, z, _, _ = oracle.quantize_pack4(Wb, 128, False)
    X = syn.activations(1, D, syn.ATTN.seed, 77, "cpu", channel_outlier_frac=0.001)
    Xb = X.view(torch.int16).numpy().view(np.uint16)
    nthreads = nthreads or oracle.default_threads()
    t0 = time.perf_counter()
    for _ in range(n_launch):
        codes = oracle.unpack4(q, D, False)
        W_hat = oracle.dequantize(codes, s, z, 128, nthreads)
        oracle.linear(Xb, W_hat, nthreads)
    dt = time.perf_counter() - t0
    return gemv_bytes(D, D, 1, False) * n_launch / dt / 1e9, nthreads, dt


def oracle_quant_sample(nthreads: int | None = None, reps: int = 1):
    """The oracle's quantize+pack and dequantize of the 4096x4096 attention
    projection (bf16 in, packed codes / bf16 out), as GB/s of the same
    algorithmic bytes the GPU numbers use."""
    import oracle
    from w4a16_bit_gemm_b200 import synthetic as syn
    W = syn.case_weight(syn.ATTN, 0, "cpu")
    Wb = W.view(torch.int16).numpy().view(np.uint16)
    nthreads = nthreads or oracle.default_threads()
    t0 = time.perf_counter()
    for _ in range(reps):
        q, s, z, _, codes = oracle.quantize_pack4(Wb, 128, False, nthreads=nthreads)
    tq = (time.perf_counter() - t0) / reps
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle.dequantize(codes, s, z, 128, nthreads)
    td = (time.perf_counter() - t0) / reps
    qb = quant_bytes(D, D, False)
    return qb / tq / 1e9, qb / td / 1e9, nthreads


def calibrated_sample(target_s: float = 12.0):
    v, n, dt = oracle_gemv_sample(1)
    per = dt
    n_launch = max(1, min(200, int(target_s / max(per, 1e-3))))
    v, n, dt = oracle_gemv_sample(n_launch)
    return v, n, dt, n_launch


def run_reference(args, dist: Dist):
    if dist.rank != 0:
        return None
    for _ in range(max(0, min(args.warmup, 1))):
        oracle_gemv_sample(1)
    v, n, dt = oracle_gemv_sample(max(1, args.steps // 200))
    n_launch = max(1, args.steps // 200)
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": v,
        "unit": "GB/s",
        "n_gpus": dist.world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": dt * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp64 accumulate over bf16 dequantized weights (CPU oracle)",
        "data": "synthetic (same seeded workload)",
        "config": {"workload": "llama7b-attn-proj W[4096,4096] g128 asym uint4, W4A16 GEMV M=1",
                   "step": f"{n_launch} oracle GEMV(s): unpack + dequantize + fp64 linear"},
        "cpu_baseline": {"value": v, "unit": "GB/s", "cores": n, "kind": "oracle",
                         "sample": f"{n_launch} GEMV launch(es) of the 4096x4096 M=1 workload"},
        "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    dist = Dist()
    try:
        if args.impl == "reference":
            out = run_reference(args, dist)
        else:
            out = run_ours(args, dist)
            if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
                v, n, dt, nl = calibrated_sample()
                v1, _, dt1 = oracle_gemv_sample(2, nthreads=1)
                qv, dv, _ = oracle_quant_sample(reps=2)
                qv1, dv1, _ = oracle_quant_sample(nthreads=1)
                out["cpu_baseline"] = {"value": v, "unit": "GB/s", "cores": n, "kind": "oracle",
                                       "sample": f"{nl} GEMV launch(es) of the 4096x4096 M=1 workload "
                                                 f"(unpack + dequantize + fp64 linear), {dt:.1f} s",
                                       "single_thread_value": v1,
                                       "single_thread_sample": f"2 launches on 1 core, {dt1:.1f} s",
                                       "quantize_GBps": qv, "dequantize_GBps": dv,
                                       "quantize_GBps_1_core": qv1, "dequantize_GBps_1_core": dv1,
                                       "quantize_sample": "quantize+pack and dequantize of W[4096,4096] g128 asym, "
                                                          f"2 reps on {n} cores, 1 rep on 1 core"}
        if out is not None and dist.rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        dist.close()


if __name__ == "__main__":
    main()
