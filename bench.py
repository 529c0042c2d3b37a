#!/usr/bin/env python
"""Benchmark of the W4A16 hot path on B200 (one JSON line on stdout, rank 0).

Workload (one "step"): the decode GEMV sweep -- M in {1, 2, 3, 4} x
N = K in {2048, 4096, 8192, 12288, 16384}, uint4 weights quantized
asymmetric with group size 128 and per channel (one group per row), bf16
activations, no bias: 40 calls of the library's GEMV through the C ABI.
Weights are quantized once with the library's own quantize-and-pack kernel
before timing ("pack once").  Calls run M-major, so each weight set is
reused only after every other set (>= 350 MB) has streamed through the
126 MB L2: the sweep's inputs are L2-cold.

The metric is whole-job HBM throughput: algorithmic bytes of the sweep
(packed weights + fp16 scales/zeros + activations + outputs) / device time.
The same sweep transposed is reported under "sweep_transposed".  Other
hot-path rows (quantize-and-pack, transposed GEMV, tensor-core GEMM forward /
transposed / with bias, fused QKV) are timed once each under "rows", and
every configuration of the workload list (the tiny case, the Llama-3.2-1B
layers in three modes with quantize-and-pack, the Llama-2-7B QLoRA layers
forward and transposed, the Llama-3-8B serving layers with bias at M = 1 ..
1024, the fractional-zero / bf16-scale variant, act-order weights) under
"configs", each against its own roofline.

Multi-GPU: one process per GPU (torchrun); each rank runs the whole sweep on
its own GPU (independent problems, no data-path collective), value = bytes
of all ranks / max-over-ranks time ("scaling": "weak").

--impl reference times the CPU oracle (the only reference this method has)
on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "W4A16 GEMM TFLOP/s and GEMV HBM GB/s vs roofline, M=1..2048, 1×B200"
SIZES = [2048, 4096, 8192, 12288, 16384]
MS = [1, 2, 3, 4]
GROUP = 128
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# --------------------------------------------------------------------- setup
def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-rows", action="store_true", help="skip the per-row table")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU baseline budget")
    ap.add_argument("--sizes", type=str, default=None, help="comma list overriding N=K sizes")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(dist, value: float, device) -> float:
    """Max of a per-rank timing over all ranks (identity without a process group)."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_value(world: int, bytes_per_step: int, ms_per_step: float) -> float:
    """Whole-job GB/s: every rank runs the full sweep, timed by the slowest rank."""
    return world * bytes_per_step / (ms_per_step * 1e-3) / 1e9


def case_bytes(M, N, K, groups_per_row, out_len=None):
    """Algorithmic bytes of one GEMV call: packed W + fp16 s,z + X + Y."""
    out_len = N if out_len is None else out_len
    in_len = K if out_len == N else N
    return N * K // 2 + 4 * N * groups_per_row + 2 * M * in_len + 2 * M * out_len


def source_hash():
    """Hash of the CUDA sources with comments and blank lines removed, so a
    comment edit does not mark committed counters as stale."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gemv_w4a16_groupwise_b200", "csrc")
    for fn in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, fn)) as f:
            text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
        lines = [re.sub(r"//.*", "", l).rstrip() for l in text.splitlines()]
        h.update(fn.encode())
        h.update("\n".join(l for l in lines if l.strip()).encode())
    return h.hexdigest()[:16]


def committed_traffic():
    """DRAM bytes of one sweep step from the committed ncu summary,
    if it was taken on the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "gemv_fwd_decode_sweep_traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    if t.get("source_hash") != source_hash():
        return None
    return t.get("dram_bytes_per_step")


# ------------------------------------------------------------- clock sampler
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------- our arm
def build_sweep(torch, w4, dev, sizes, seed=1234):
    """Quantize the sweep's weight sets on the device; returns the case list."""
    gen = torch.Generator(device=dev)
    sets = []
    for N in sizes:
        K = N
        gen.manual_seed(seed + N)
        W = (torch.randn((N, K), generator=gen, device=dev, dtype=torch.float32) * 0.02).to(torch.bfloat16)
        for mode, g in (("groupwise", GROUP), ("rowwise", 0)):
            p, s, z = w4.w4_quantize_pack(W, mode, g)
            sets.append(dict(N=N, K=K, mode=mode, g=g, p=p, s=s, z=z,
                             G=(K // g if mode == "groupwise" else 1)))
        del W
    torch.cuda.synchronize(dev)
    cases = []
    for M in MS:                     # M-major: a set is reused only after all the others
        for ws in sets:
            gen.manual_seed(seed + 7 * M + ws["N"])
            X = torch.randn((M, ws["K"]), generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16)
            Y = torch.empty((M, ws["N"]), dtype=torch.bfloat16, device=dev)
            dY = torch.randn((M, ws["N"]), generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16)
            dX = torch.empty((M, ws["K"]), dtype=torch.bfloat16, device=dev)
            nws = w4.w4_workspace_bytes(M, ws["N"], ws["K"], False)
            nws_t = w4.w4_workspace_bytes(M, ws["N"], ws["K"], True)
            cases.append(dict(M=M, set=ws, X=X, Y=Y, dY=dY, dX=dX, nws=nws, nws_t=nws_t,
                              bytes=case_bytes(M, ws["N"], ws["K"], ws["G"]),
                              bytes_t=case_bytes(M, ws["N"], ws["K"], ws["G"], out_len=ws["K"])))
    max_ws = max(max(c["nws"], c["nws_t"]) for c in cases)
    wsbuf = torch.empty(max(max_ws, 16), dtype=torch.uint8, device=dev)
    return cases, wsbuf


def make_step(w4, cases, wsbuf, stream_ptr, transposed=False):
    lib = w4.library()
    xk, yk, nk = ("dY", "dX", "nws_t") if transposed else ("X", "Y", "nws")

    def step():
        for c in cases:
            s = c["set"]
            st = lib.w4a16_gemv(c[xk].data_ptr(), c["M"], s["N"], s["K"], s["p"].data_ptr(),
                                s["s"].data_ptr(), s["z"].data_ptr(), w4.MODES[s["mode"]], s["g"],
                                None, 1 if transposed else 0, c[yk].data_ptr(), wsbuf.data_ptr(), c[nk],
                                stream_ptr())
            if st != 0:
                raise RuntimeError(f"w4a16_gemv failed: {lib.w4_status_string(st).decode()}")
    return step


def time_graph(torch, graph, reps, stream):
    # CUDAGraph.replay() launches on the current stream: make it the timed one
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def capture(torch, fn, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        fn()  # warm (also sets kernel attributes outside capture)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=stream):
            fn()
    torch.cuda.synchronize()
    return g


def flush_l2(torch, buf):
    buf.add_(1)


def measure_rows(torch, w4, dev, peaks, stream):
    """One timing per remaining hot-path row, L2 flushed before each launch."""
    rows = {}
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(99)

    def rnd(shape, std=1.0):
        return (torch.randn(shape, generator=gen, device=dev, dtype=torch.float32) * std).to(torch.bfloat16)

    def timed(fn, reps=5):
        ts = []
        for _ in range(reps):
            flush_l2(torch, flush)
            # keep the GPU busy (no memory traffic) while the host enqueues
            # the call, so the events bracket device time only
            torch.cuda._sleep(1_000_000)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return statistics.median(ts)

    with torch.cuda.stream(stream):
        # quantize + pack, Llama-3.2-1B lm-head shape, groupwise g=64
        N, K = 128256, 2048
        W = rnd((N, K), 0.02)
        w4.w4_quantize_pack(W, "groupwise", 64)
        ms = timed(lambda: w4.w4_quantize_pack(W, "groupwise", 64))
        qb = 2 * N * K + N * K // 2 + 4 * N * (K // 64)
        rows["quantize_pack"] = {"shape": "N=128256 K=2048 g=64", "us": ms * 1e3,
                                 "GB/s": qb / ms / 1e6, "frac_hbm": qb / ms / 1e6 / peaks["hbm_gbs"]}
        P, S, Z = w4.w4_quantize_pack(W, "groupwise", 64)
        del W
        # GEMM forward at the same shape, M = 2048
        for M in (128, 512, 2048):
            X = rnd((M, K))
            w4.w4a16_gemm(X, P, S, Z, "groupwise", 64, N=N, K=K)
            ms = timed(lambda: w4.w4a16_gemm(X, P, S, Z, "groupwise", 64, N=N, K=K), reps=3)
            tf = 2.0 * M * N * K / ms / 1e9
            rows[f"gemm_fwd_M{M}"] = {"shape": f"M={M} N=128256 K=2048 g=64", "us": ms * 1e3,
                                      "TFLOP/s": tf, "frac_bf16": tf / peaks["bf16_tflops"]}
        del P, S, Z
        # transposed GEMM and fused QKV, Llama-2-7B QLoRA shapes, M = 2048
        N, K, M = 11008, 4096, 2048
        W = rnd((N, K), 0.02)
        P, S, Z = w4.w4_quantize_pack(W, "groupwise", 64)
        dY = rnd((M, N))
        w4.w4a16_gemm(dY, P, S, Z, "groupwise", 64, N=N, K=K, transposed=True)
        ms = timed(lambda: w4.w4a16_gemm(dY, P, S, Z, "groupwise", 64, N=N, K=K, transposed=True))
        tf = 2.0 * M * N * K / ms / 1e9
        rows["gemm_t_M2048"] = {"shape": "M=2048 N=11008 K=4096 g=64 transposed", "us": ms * 1e3,
                                "TFLOP/s": tf, "frac_bf16": tf / peaks["bf16_tflops"]}
        X = rnd((M, K))
        ms = timed(lambda: w4.w4a16_gemm(X, P, S, Z, "groupwise", 64, N=N, K=K))
        tf = 2.0 * M * N * K / ms / 1e9
        rows["gemm_fwd_M2048_llama2_up"] = {"shape": "M=2048 N=11008 K=4096 g=64", "us": ms * 1e3,
                                            "TFLOP/s": tf, "frac_bf16": tf / peaks["bf16_tflops"]}
        del W, P, S, Z
        N = 3 * 4096
        W = rnd((N, 4096), 0.02)
        P, S, Z = w4.w4_quantize_pack(W, "groupwise", 64)
        X = rnd((M, 4096))
        dY = rnd((M, N))
        ms_f = timed(lambda: w4.w4a16_gemm(X, P, S, Z, "groupwise", 64, N=N, K=4096))
        ms_t = timed(lambda: w4.w4a16_gemm(dY, P, S, Z, "groupwise", 64, N=N, K=4096, transposed=True))
        fl = 2.0 * M * N * 4096
        rows["fused_qkv_M2048"] = {"shape": "M=2048 N=3x4096 K=4096 g=64",
                                   "fwd_TFLOP/s": fl / ms_f / 1e9, "t_TFLOP/s": fl / ms_t / 1e9}
        del W, P, S, Z
        # bias epilogue, Llama-3-8B gate_up, M = 1024, g = 128
        N, K, M = 28672, 4096, 1024
        W = rnd((N, K), 0.02)
        P, S, Z = w4.w4_quantize_pack(W, "groupwise", 128)
        X = rnd((M, K))
        b = rnd((N,), 0.01)
        ms = timed(lambda: w4.w4a16_gemm(X, P, S, Z, "groupwise", 128, N=N, K=K, bias=b))
        tf = 2.0 * M * N * K / ms / 1e9
        rows["gemm_bias_M1024"] = {"shape": "M=1024 N=28672 K=4096 g=128 +bias", "us": ms * 1e3,
                                   "TFLOP/s": tf, "frac_bf16": tf / peaks["bf16_tflops"]}
        # transposed GEMV, M = 4
        dY4 = rnd((4, N))
        ms = timed(lambda: w4.w4a16_gemv(dY4, P, S, Z, "groupwise", 128, N=N, K=K, transposed=True))
        gb = case_bytes(4, N, K, K // 128, out_len=K) / ms / 1e6
        rows["gemv_t_M4"] = {"shape": "M=4 N=28672 K=4096 g=128 transposed", "us": ms * 1e3,
                             "GB/s": gb, "frac_hbm": gb / peaks["hbm_gbs"]}
        del W, P, S, Z, flush
    torch.cuda.synchronize()
    return rows


def gemm_roofline(M, N, K, G, peaks, bias=False, out_len=None):
    """Algorithmic work of one call and the time it needs at the measured
    peaks: the slower of the tensor-core time for 2 M N K flops and the HBM
    time for the packed weights, scales, zeros, activations and outputs."""
    flops = 2.0 * M * N * K
    byts = case_bytes(M, N, K, G, out_len=out_len) + (2 * (out_len or N) if bias else 0)
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    t_hbm = byts / (peaks["hbm_gbs"] * 1e9)
    return flops, byts, ("tensor" if t_tc >= t_hbm else "hbm"), max(t_tc, t_hbm)


def measure_configs(torch, w4, dev, peaks, stream):
    """Every configuration of the workload list, one timed call each (L2
    flushed before it): the tiny correctness case, the Llama-3.2-1B layers in
    three quantization modes with quantize-and-pack of each weight, the
    Llama-2-7B QLoRA layers forward and transposed, the Llama-3-8B serving
    layers with bias at M = 1 .. 1024, the fractional-zero variant (fp16
    and bf16 metadata) and act-order weights on decode and training shapes.  Each row reports the
    fraction of its own roofline (the slower of tensor-core and HBM time)."""
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(7)

    def rnd(shape, std=1.0):
        return (torch.randn(shape, generator=gen, device=dev, dtype=torch.float32) * std).to(torch.bfloat16)

    def timed(fn, reps=3):
        fn()
        ts = []
        for _ in range(reps):
            flush_l2(torch, flush)
            torch.cuda._sleep(1_000_000)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return statistics.median(ts) * 1e-3          # seconds

    def row(name, M, N, K, mode, g, fn, transposed=False, bias=False):
        G = 1 if mode != "groupwise" else K // g
        t = timed(fn)
        out_len = K if transposed else N
        flops, byts, bound, t_min = gemm_roofline(M, N, K, G, peaks, bias=bias, out_len=out_len)
        return {"case": name, "M": M, "N": N, "K": K, "mode": mode, "g": g, "transposed": transposed,
                "bias": bias, "us": round(t * 1e6, 2), "TFLOP/s": round(flops / t / 1e12, 2),
                "GB/s": round(byts / t / 1e9, 1), "bound": bound, "frac": round(t_min / t, 4)}

    out = {}
    with torch.cuda.stream(stream):
        # tiny correctness case: M = 4, N = 256, K = 512, g = 64, forward and transposed
        N, K, g = 256, 512, 64
        W = rnd((N, K), 0.02)
        P, S, Z = w4.w4_quantize_pack(W, "groupwise", g)
        X, dY = rnd((4, K)), rnd((4, N))
        out["config1_tiny"] = [
            row("tiny fwd", 4, N, K, "groupwise", g, lambda: w4.w4a16_gemv(X, P, S, Z, "groupwise", g, N=N, K=K)),
            row("tiny t", 4, N, K, "groupwise", g,
                lambda: w4.w4a16_gemv(dY, P, S, Z, "groupwise", g, N=N, K=K, transposed=True), transposed=True)]
        # Llama-3.2-1B layers: three modes, M = 128, 512, 2048, and quantize + pack of each W
        rows, qrows = [], []
        for (N, K) in ((2048, 2048), (8192, 2048), (2048, 8192), (512, 2048), (128256, 2048)):
            W = rnd((N, K), 0.02)
            for mode, g in (("global", 0), ("rowwise", 0), ("groupwise", 64)):
                G = 1 if mode != "groupwise" else K // g
                t = timed(lambda: w4.w4_quantize_pack(W, mode, g))
                qb = 2 * N * K + N * K // 2 + 4 * N * G + (2 * N * K if mode == "global" else 0)
                qrows.append({"N": N, "K": K, "mode": mode, "g": g, "us": round(t * 1e6, 2),
                              "GB/s": round(qb / t / 1e9, 1),
                              "frac": round(qb / t / 1e9 / peaks["hbm_gbs"], 4)})
                P, S, Z = w4.w4_quantize_pack(W, mode, g)
                for M in (128, 512, 2048):
                    X = rnd((M, K))
                    rows.append(row("llama3.2-1b", M, N, K, mode, g,
                                    lambda: w4.w4a16_gemm(X, P, S, Z, mode, g, N=N, K=K)))
                del P, S, Z
            del W
        out["config3_llama32_1b"] = rows
        out["config3_quantize_pack"] = qrows
        # Llama-2-7B QLoRA layers: forward and transposed, g = 64 and per channel
        rows = []
        for (N, K) in ((3 * 4096, 4096), (4096, 4096), (11008, 4096), (4096, 11008)):
            W = rnd((N, K), 0.02)
            for mode, g in (("groupwise", 64), ("rowwise", 0)):
                P, S, Z = w4.w4_quantize_pack(W, mode, g)
                for M in (1024, 2048):
                    X, dY = rnd((M, K)), rnd((M, N))
                    rows.append(row("llama2-7b fwd", M, N, K, mode, g,
                                    lambda: w4.w4a16_gemm(X, P, S, Z, mode, g, N=N, K=K)))
                    rows.append(row("llama2-7b t", M, N, K, mode, g,
                                    lambda: w4.w4a16_gemm(dY, P, S, Z, mode, g, N=N, K=K, transposed=True),
                                    transposed=True))
                del P, S, Z
            del W
        out["config4_llama2_7b"] = rows
        # Llama-3-8B serving layers with bias, g = 128, M = 1 .. 1024
        rows = []
        for (N, K) in ((6144, 4096), (4096, 4096), (28672, 4096), (4096, 14336)):
            W = rnd((N, K), 0.02)
            P, S, Z = w4.w4_quantize_pack(W, "groupwise", 128)
            b = rnd((N,), 0.01)
            for M in (1, 4, 16, 64, 256, 1024):
                X = rnd((M, K))
                rows.append(row("llama3-8b", M, N, K, "groupwise", 128,
                                lambda: w4.w4a16_gemm(X, P, S, Z, "groupwise", 128, N=N, K=K, bias=b), bias=True))
            del W, P, S, Z
        out["config5_llama3_8b_bias"] = rows
        # the HQQ-style variant: fractional zero point, fp16 and bf16 scales / zeros,
        # quantize + pack and the decode / training products on the same shapes
        rows = []
        for (N, K, g) in ((16384, 16384, 128), (8192, 8192, 128), (11008, 4096, 64)):
            W = rnd((N, K), 0.02)
            for meta in ("fp16", "bf16"):
                t = timed(lambda: w4.w4_quantize_pack(W, "groupwise", g, zero="float", meta=meta))
                qb = 2 * N * K + N * K // 2 + 4 * N * (K // g)
                rows.append({"case": f"quantize float-zero {meta}", "N": N, "K": K, "g": g, "us": round(t * 1e6, 2),
                             "GB/s": round(qb / t / 1e9, 1), "frac": round(qb / t / 1e9 / peaks["hbm_gbs"], 4)})
                P, S, Z = w4.w4_quantize_pack(W, "groupwise", g, zero="float", meta=meta)
                Ms = (1, 4) if N == K else (2048,)
                for M in Ms:
                    X, dY = rnd((M, K)), rnd((M, N))
                    r = row(f"float-zero {meta} fwd", M, N, K, "groupwise", g,
                            lambda: w4.w4a16_gemm(X, P, S, Z, "groupwise", g, N=N, K=K, zero="float"))
                    rows.append(r)
                    r = row(f"float-zero {meta} t", M, N, K, "groupwise", g,
                            lambda: w4.w4a16_gemm(dY, P, S, Z, "groupwise", g, N=N, K=K, transposed=True,
                                                  zero="float"), transposed=True)
                    rows.append(r)
                del P, S, Z
            del W
        out["variant_float_zero"] = rows
        # act-order weights (packed column j = input channel perm[j]): the gather of
        # X's columns (forward) or the scatter of dX's (transposed) is inside the call
        rows = []
        for (N, K, g, Ms) in ((8192, 8192, 128, (1, 4)), (11008, 4096, 64, (2048,))):
            W = rnd((N, K), 0.02)
            perm = torch.randperm(K, generator=gen, device=dev).to(torch.int32)
            P, S, Z = w4.w4_quantize_pack(W, "groupwise", g, perm=perm)
            for M in Ms:
                X, dY = rnd((M, K)), rnd((M, N))
                rows.append(row("act-order fwd", M, N, K, "groupwise", g,
                                lambda: w4.w4a16_gemm(X, P, S, Z, "groupwise", g, N=N, K=K, perm=perm)))
                rows.append(row("act-order t", M, N, K, "groupwise", g,
                                lambda: w4.w4a16_gemm(dY, P, S, Z, "groupwise", g, N=N, K=K, transposed=True,
                                                      perm=perm), transposed=True))
            del W, P, S, Z
        out["variant_act_order"] = rows
        del flush
    torch.cuda.synchronize()
    return out


def host_cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def single_thread_oracle(sizes):
    """The oracle on one host thread: the tiny correctness case (whole) and
    one call of the decode sweep per N = K (64 output rows, M = 4)."""
    code = (
        "import time, json, oracle\n"
        "from gemv_w4a16_groupwise_b200 import synth\n"
        "res = {}\n"
        "W = synth.weights(256, 512, 0); p, s, z = oracle.quantize_pack(W, 'groupwise', 64)\n"
        "X = synth.activations(4, 512, 0); t0 = time.perf_counter()\n"
        "oracle.linear(X, p, s, z, 'groupwise', 64, 256, 512)\n"
        "res['tiny_fwd_s'] = time.perf_counter() - t0\n"
        f"for N in {list(sizes)}:\n"
        "    W = synth.weights(64, N, 1); p, s, z = oracle.quantize_pack(W, 'groupwise', 128)\n"
        "    X = synth.activations(4, N, 1); t0 = time.perf_counter()\n"
        "    oracle.linear(X, p, s, z, 'groupwise', 128, 64, N)\n"
        "    dt = time.perf_counter() - t0\n"
        "    res[f'sweep_M4_N{N}_64rows_s'] = dt\n"
        "print(json.dumps(res))\n")
    env = dict(os.environ, OMP_NUM_THREADS="1")
    try:
        r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True,
                           timeout=120)
        return json.loads(r.stdout.strip().splitlines()[-1])
    except (subprocess.SubprocessError, ValueError, IndexError):
        return None


def cpu_baseline(seconds_budget, sizes):
    """The oracle, as it stands, on a bounded sample of the sweep: for every
    case it computes R output columns (R sampled weight rows, quantized by the
    oracle) for all M; R is calibrated to the time budget."""
    import oracle
    from gemv_w4a16_groupwise_b200 import synth
    threads = oracle.num_threads()

    def run(R):
        total_b, total_t = 0, 0.0
        for N in sizes:
            K = N
            rows = min(N, R)
            seed = synth.config_seed("cpu", N)
            Wr = synth.weights(rows, K, seed)
            for mode, g in (("groupwise", GROUP), ("rowwise", 0)):
                p, s_, z = oracle.quantize_pack(Wr, mode, g)
                G = K // g if mode == "groupwise" else 1
                for M in MS:
                    X = synth.activations(M, K, seed + M)
                    t0 = time.perf_counter()
                    oracle.linear(X, p, s_, z, mode, g, rows, K)
                    total_t += time.perf_counter() - t0
                    total_b += case_bytes(M, rows, K, G)
        return total_b, total_t

    _, t0 = run(32)
    R = int(max(32, min(8192, 32 * seconds_budget / max(t0, 1e-3))))
    b, t = run(R)
    return {"value": b / t / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"all {8 * len(sizes)} sweep cases, min(N, {R}) output rows each (fp64 C oracle, OpenMP)",
            "seconds": round(t, 3)}


def run_ours(args):
    import torch
    import gemv_w4a16_groupwise_b200 as w4

    ws_, rank, local = dist_env()
    dist = None
    if ws_ > 1:
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    sizes = [int(s) for s in args.sizes.split(",")] if args.sizes else SIZES

    stream = torch.cuda.Stream(dev)
    stream_ptr = lambda: __import__("ctypes").c_void_p(stream.cuda_stream)
    cases, wsbuf = build_sweep(torch, w4, dev, sizes)
    step = make_step(w4, cases, wsbuf, stream_ptr)
    bytes_step = sum(c["bytes"] for c in cases)

    n0 = w4.w4_launch_count()
    with torch.cuda.stream(stream):
        step()
    torch.cuda.synchronize()
    launches_per_step = w4.w4_launch_count() - n0
    graph = capture(torch, step, stream)
    sampler = ClockSampler(local)
    with torch.cuda.stream(stream):        # replay() launches on the current stream
        for _ in range(max(3, args.warmup)):
            graph.replay()
        torch.cuda.synchronize()
        sampler.start()
        t_end = time.time() + 0.6
        while time.time() < t_end:         # let the sampler see the load
            graph.replay()
            torch.cuda.synchronize()
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        ms_step = e0.elapsed_time(e1) / args.steps
        t_end = time.time() + 0.3
        while time.time() < t_end:
            graph.replay()
            torch.cuda.synchronize()
    clocks = sampler.stop()
    ms_step = max_over_ranks(dist, ms_step, dev)
    value = weak_value(ws_, bytes_step, ms_step)

    # the same sweep, transposed (dX = dY . dequant(W)), timed the same way
    step_t = make_step(w4, cases, wsbuf, stream_ptr, transposed=True)
    graph_t = capture(torch, step_t, stream)
    with torch.cuda.stream(stream):
        for _ in range(3):
            graph_t.replay()
    ms_t = time_graph(torch, graph_t, max(10, args.steps // 3), stream)
    bytes_t = sum(c["bytes_t"] for c in cases)
    sweep_t = {"GB/s": round(bytes_t / (ms_t * 1e-3) / 1e9, 2),
               "frac": round(bytes_t / (ms_t * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
               "ms_per_step": round(ms_t, 5), "calls": len(cases),
               "workload": "the decode sweep transposed: dY [M, N] -> dX [M, K], same weights"}
    del graph_t

    # per-case device times (20 back-to-back calls of one case; L2 warm for the
    # small sets -- reported for context, the headline is the cold sweep).
    # The 20 calls sit in one graph, so the host's launch rate does not
    # limit the short ones.
    per_case = []
    for c in cases:
        one = make_step(w4, [c] * 20, wsbuf, stream_ptr)
        g1 = capture(torch, one, stream)
        msc = time_graph(torch, g1, 3, stream) / 20
        per_case.append({"M": c["M"], "N": c["set"]["N"], "K": c["set"]["K"], "mode": c["set"]["mode"],
                         "us": round(msc * 1e3, 2), "GB/s": round(c["bytes"] / msc / 1e6, 1),
                         "frac": round(c["bytes"] / msc / 1e6 / peaks["hbm_gbs"], 4)})
        del g1

    # end to end through the public API with host buffers: the step's
    # activations sit in one pinned host buffer and reach the device in one
    # copy, each call reads its slice (every slice starts on a 16-byte
    # boundary: M * K and M * N are multiples of 8), and the step's outputs
    # come back in one copy.  Copies of a few kilobytes each, in order
    # between the calls, would put a DMA latency per call on the path.
    nx = [c["X"].numel() for c in cases]
    ny = [c["Y"].numel() for c in cases]
    ox = [sum(nx[:i]) for i in range(len(cases))]
    oy = [sum(ny[:i]) for i in range(len(cases))]
    pinned_x = torch.empty(sum(nx), dtype=torch.bfloat16).pin_memory()
    for c, o, n in zip(cases, ox, nx):
        pinned_x[o:o + n].copy_(c["X"].reshape(-1).cpu())
    pinned_y = torch.empty(sum(ny), dtype=torch.bfloat16).pin_memory()
    dev_xall = torch.empty(sum(nx), dtype=torch.bfloat16, device=dev)
    dev_yall = torch.empty(sum(ny), dtype=torch.bfloat16, device=dev)
    dev_x = [dev_xall[o:o + n].view(c["X"].shape) for c, o, n in zip(cases, ox, nx)]
    dev_y = [dev_yall[o:o + n].view(c["Y"].shape) for c, o, n in zip(cases, oy, ny)]
    h2d = pinned_x.numel() * 2
    d2h = pinned_y.numel() * 2

    def e2e_step():
        dev_xall.copy_(pinned_x, non_blocking=True)
        for i, c in enumerate(cases):
            s = c["set"]
            w4.w4a16_gemv(dev_x[i], s["p"], s["s"], s["z"], s["mode"], s["g"], N=s["N"], K=s["K"],
                          out=dev_y[i])
        pinned_y.copy_(dev_yall, non_blocking=True)

    e2e_steps = max(3, min(args.steps, 30))
    with torch.cuda.stream(stream):
        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        a1.record(stream)
        torch.cuda.synchronize()
    ms_e2e = max_over_ranks(dist, a0.elapsed_time(a1) / e2e_steps, dev)
    e2e_value = weak_value(ws_, bytes_step, ms_e2e)

    rows = configs = None
    if not args.no_rows:
        rows = measure_rows(torch, w4, dev, peaks, stream)
        configs = measure_configs(torch, w4, dev, peaks, stream)
    del graph

    err = w4.w4_device_error()
    out = None
    if rank == 0:
        cpu = None
        if ws_ == 1 and not args.no_cpu:
            cpu = cpu_baseline(args.cpu_seconds, sizes)
            cpu["cpu_model"] = host_cpu_model()
            cpu["single_thread"] = single_thread_oracle(sizes)
        calls = len(cases)
        alg_per_call = bytes_step / calls
        traffic = committed_traffic()
        out = {
            "metric": METRIC,
            "value": round(value, 2),
            "unit": "GB/s",
            "n_gpus": ws_,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms_step, 5),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "f32",
            "operands": "uint4 weights (fp16 group scale/zero), bf16 activations and outputs, fp32 accumulation",
            "data": "synthetic (seeded torch RNG on the device: W ~ N(0, 0.02), X ~ N(0, 1))",
            "config": {
                "workload": "decode GEMV sweep: M in {1,2,3,4} x N=K in {" + ",".join(map(str, sizes)) +
                            "}, uint4 g=128 and per-channel, no bias (40 calls per step)",
                "l2": "cold: M-major call order, each weight set reused only after every other set "
                      "(>= 350 MB) streamed through the 126 MB L2",
                "timing": "CUDA graph of one step, CUDA events on the launching stream",
                "parallelism": f"replicated sweep per rank (weak), {ws_} rank(s)",
            },
            "roofline": {
                "bound": "hbm",
                "achieved": round(alg_per_call / (ms_step / calls * 1e-3) / 1e9, 2),
                "peak": peaks["hbm_gbs"],
                "unit": "GB/s",
                "frac": round(alg_per_call / (ms_step / calls * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                "traffic": (round(traffic / calls) if traffic is not None else None),
                "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured"
                               else "fallback 6.65 TB/s",
                "kernel": "gemv_q8_kernel (one launch per GEMV call in this sweep: no shape splits K)",
                "per": "GEMV call, averaged over the 40 calls of a step (CUDA events on the launching "
                       "stream around the whole timed region)",
                "alg_bytes_per_launch": round(alg_per_call),
                "traffic_source": "profiles/gemv_fwd_decode_sweep_traffic.json (ncu dram__bytes_read.sum + "
                                  "dram__bytes_write.sum of both kernels, one step; null when the kernel "
                                  "sources changed since)",
            },
            "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h,
                    "path": "the step's X (one pinned host buffer) -> device in one copy, 40 w4a16_gemv calls "
                            "through the Python binding on its slices, the step's Y -> pinned host in one copy; "
                            "eager"},
            "gpu_launches": int(launches_per_step * args.steps),
            "launches_per_step": int(launches_per_step),
            "clocks": clocks,
            "cpu_baseline": cpu,
            "device_error_word": err,
            "cases": per_case,
            "sweep_transposed": sweep_t,
            "rows": rows,
            "configs": configs,
        }
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return out


# ------------------------------------------------------------ reference arm
def run_reference(args):
    ws_, rank, _ = dist_env()
    if rank != 0:
        return None
    sizes = [int(s) for s in args.sizes.split(",")] if args.sizes else SIZES
    per_step_budget = max(1.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_baseline(per_step_budget / 4, sizes)
    vals, secs = [], 0.0
    last = None
    for _ in range(args.steps):
        last = cpu_baseline(per_step_budget, sizes)
        vals.append(last["value"])
        secs += last["seconds"]
    value = statistics.median(vals)
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 4),
        "unit": "GB/s",
        "n_gpus": ws_,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(1e3 * secs / max(1, args.steps), 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded numpy PCG64: W ~ N(0, 0.02), X ~ N(0, 1))",
        "config": {"workload": "decode GEMV sweep (bounded sample: every case, a subset of output rows)"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": last["cores"],
                         "kind": "oracle", "sample": last["sample"]},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse_args()
    out = run_reference(args) if args.impl == "reference" else run_ours(args)
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
