#!/usr/bin/env python
"""Benchmark of the LLM.int8() Linear8bitLt forward hot path on B200.

One step = one forward pass of every linear of the workload (default: the seven
linears of a Llama-7B-shaped decoder layer at 4096 prefill tokens), each
linear = fused quantise + outlier prepare + tcgen05 int8 GEMM with the fused
dequant / bias / fp16-outlier epilogue.  Inputs are resident in HBM when the
timed region starts; weights are quantised once before it (load time).

Prints ONE JSON line (rank 0).  ``--impl reference`` times the CPU oracle on a
bounded row sample of the same workload instead (the slow reference arm).

Multi-GPU: the path has no exchange step, so ``--gpus N`` under torchrun runs N
independent replicas (weak scaling, no data-path collective); the timed region
is bracketed by barriers and the slowest rank's device time is reported.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from int8_mixed_precision_vectorwise_b200 import workloads as wl  # noqa: E402

METRIC = "LLM.int8() linear TOPS (2MNK/s) vs int8 TC peak; decode weight-read GB/s"
MAX_OUTLIER_COLS = 256
GEMM_SOURCES = ("int8_mixed_precision_vectorwise_b200/csrc/gemm_tcgen05.cu",
                "int8_mixed_precision_vectorwise_b200/csrc/ptx.cuh")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "gemm_tcgen05_llama7b_prefill_traffic.txt")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="C3")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--no-other", action="store_true", help="skip the single-linear, OPT MLP and outlier sweep")
    ap.add_argument("--no-shared", action="store_true", help="skip the shared-input layer step")
    ap.add_argument("--no-quant", action="store_true", help="skip the quantiser roofline")
    ap.add_argument("--no-nf4", action="store_true", help="skip the NF4 decode product")
    ap.add_argument("--cpu-rows", type=int, default=256, help="rows per linear in the CPU oracle sample")
    return ap.parse_args()


def describe(W: wl.Workload) -> str:
    parts = [f"{L.name} {L.M}x{L.K}->{L.N}" + (f" ({L.n_out} outlier cols U{L.mag})" if L.n_out else "")
             for L in W.layers]
    return f"{W.key}: " + "; ".join(parts) + f"; threshold {W.layers[0].threshold:g}"


def gemm_source_sha() -> str:
    h = hashlib.sha256()
    for f in GEMM_SOURCES:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()[:16]


def read_traffic():
    """Per-launch DRAM bytes of the GEMM from the committed ncu summary, if it
    was taken on the current kernel source; else None."""
    try:
        kv = dict(l.strip().split("=", 1) for l in open(TRAFFIC_FILE) if "=" in l and not l.startswith("#"))
        if kv.get("kernel_sha") == gemm_source_sha():
            return float(kv["dram_bytes_per_launch"])
    except (OSError, ValueError, KeyError):
        pass
    return None


def measured_peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except OSError:
        return None


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch_device):
        self.samples = []
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(torch_device).uuid)
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001
            self.err = repr(e)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM),
                                     nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": getattr(self, "err", "no NVML")}
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = [s[0] for s in self.samples]
        mask = 0
        for _, r in self.samples:
            mask |= int(r)
        return {"sm_mhz": float(statistics.median(mhz)), "sm_max_mhz": self.max_mhz,
                "reasons": [n for b, n in self.REASONS.items() if mask & b], "samples": len(mhz),
                "sm_mhz_min": min(mhz)}


# ------------------------------------------------------------------ multi-rank helpers
def max_over_ranks(x: float, world: int, dist, device) -> float:
    """The largest x over all ranks: a job's time is its slowest rank's time."""
    if world <= 1:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(ops_per_step: float, steps: int, world: int, ms: float) -> float:
    """Whole-job TOPS: every rank (a replica) runs `steps` steps of `ops_per_step`
    operations; the job takes `ms`, the time of its slowest rank."""
    return world * ops_per_step * steps / (ms / 1e3) / 1e12


def nearest_rank(xs, ps):
    """Nearest-rank percentiles (p in [0, 1]) of a non-empty sample: the ceil(p * n)-th
    smallest value (the smallest one for p = 0)."""
    import math
    v = sorted(xs)
    return [v[min(len(v) - 1, max(0, math.ceil(p * len(v)) - 1))] for p in ps]


# ------------------------------------------------------------------ CPU oracle timing
def cpu_oracle_steps(layers_np, rows: int, steps: int, min_seconds: float = 0.0):
    """Run the oracle forward on the first `rows` rows of every linear; returns (seconds per step, ops per step)."""
    import oracle
    ops = sum(2 * min(rows, X.shape[0]) * CB.shape[0] * X.shape[1] for X, CB, _, _, _ in layers_np)
    times = []
    t_all = time.perf_counter()
    k = 0
    while k < steps or (time.perf_counter() - t_all) < min_seconds:
        t0 = time.perf_counter()
        for X, CB, SCB, b, tau in layers_np:
            oracle.linear8bit_forward(X[:rows], CB, SCB, b, tau)
        times.append(time.perf_counter() - t0)
        k += 1
    return times, ops


def decode_bytes(L) -> int:
    """Algorithmic bytes of one few-token forward: the int8 weight, its scales, X and out."""
    return L.N * L.K + 4 * L.N + 2 * L.M * L.K + 2 * L.M * L.N


def graph_us(torch, dev, st, fn, calls: int, replays: int = 3) -> float:
    """Device time per call of `fn` with the host out of the way: `calls` calls captured in one
    CUDA graph, replayed `replays` times between CUDA events on `st` after one warm-up replay.
    A call whose host side (argument checks, the C entry, the launches) takes longer than its
    kernels leaves the GPU idle between back-to-back eager calls; the replay does not."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(calls):
            fn()
    g.replay()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(replays):
        g.replay()
    e1.record(st)
    torch.cuda.synchronize(dev)
    us = e0.elapsed_time(e1) / (replays * calls) * 1e3
    del g
    return us


def measure_decode(i8, torch, dev, st, world, dist, reps: int = 20):
    """Every point of the decode grid (tokens {1, 4, 16} x outlier columns {0, 1, 8}) on both
    Llama-70B FFN shapes.  Weights (235 MB each, > L2) stream from HBM every call.  Per point:
    the whole forward (preparation + few-token GEMM, launched as in production, `reps`
    back-to-back calls), then a second pass with events between the two kernels, which gives
    the preparation alone and the GEMM alone (each then starts without the other's overlap)."""
    W = wl.workloads()
    points = []
    hbm = (measured_peaks() or {}).get("hbm_gbs", 6650.0)
    weights = {}
    keys = [f"C4_t{t}_o{o}" for t in (1, 4, 16) for o in (0, 1, 8)]
    for key in keys:
        for li, L in enumerate(W[key].layers):
            wk = (L.N, L.K)
            if wk not in weights:
                _, _, Wt, _ = wl.layer_inputs(wl.seed_of("C4_t1_o0"), li, L)
                CB, SCB, _ = i8.i8_quantize_rowwise(torch.from_numpy(Wt).to(dev), 0.0)
                weights[wk] = (CB, SCB)
            CB, SCB = weights[wk]
            X, _, _, _ = wl.layer_inputs(wl.seed_of(key), li, L)
            dX = torch.from_numpy(X).to(dev)
            out = torch.empty((L.M, L.N), dtype=torch.float16, device=dev)
            ws = torch.empty((i8.i8_linear8bit_workspace_size(L.M, L.N, L.K, MAX_OUTLIER_COLS),),
                             dtype=torch.uint8, device=dev)

            def fwd():
                i8.i8_linear8bit_forward(dX, CB, SCB, None, L.threshold, out=out, workspace=ws,
                                         max_outlier_cols=MAX_OUTLIER_COLS)
            for _ in range(3):
                fwd()
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize(dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(st)
            for _ in range(reps):
                fwd()
            e1.record(st)
            torch.cuda.synchronize(dev)
            ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(reps)]
            for r in range(reps):
                ev[r][0].record(st)
                i8.i8_linear8bit_prepare(dX, CB, L.threshold, ws, MAX_OUTLIER_COLS)
                ev[r][1].record(st)
                i8.i8_linear8bit_matmul_dequant(CB, SCB, None, L.M, L.threshold, out, ws, MAX_OUTLIER_COLS)
                ev[r][2].record(st)
            torch.cuda.synchronize(dev)
            us_graph = graph_us(torch, dev, st, fwd, reps)
            code, _ = i8.i8_read_status(ws)
            if code != 0:
                raise RuntimeError(f"decode status {i8.STATUS.get(code, code)}")
            us = e0.elapsed_time(e1) / reps * 1e3
            prep_us = sum(a.elapsed_time(b) for a, b, _ in ev) / reps * 1e3
            gemm_us = sum(b.elapsed_time(c) for _, b, c in ev) / reps * 1e3
            gbs = decode_bytes(L) / us / 1e3
            points.append({"shape": f"{L.M}x{L.K}->{L.N}", "tokens": L.M, "outlier_cols": L.n_out,
                           "us": round(us, 2), "GB/s": round(gbs, 1), "frac": round(gbs / hbm, 4),
                           "us_graph": round(us_graph, 2),
                           "frac_graph": round(decode_bytes(L) / us_graph / 1e3 / hbm, 4),
                           "prep_alone_us": round(prep_us, 2), "gemm_alone_us": round(gemm_us, 2),
                           "gemm_alone_frac": round(decode_bytes(L) / gemm_us / 1e3 / hbm, 4)})
    best = max(points, key=lambda q: q["GB/s"])
    worst = min(points, key=lambda q: q["GB/s"])
    return {"metric": "decode weight-read GB/s (whole forward per call)", "peak_gbs": hbm,
            "timing": f"us: CUDA events over {reps} back-to-back eager calls; us_graph: the same calls "
                      "replayed from a CUDA graph (no host time between forwards)",
            "peak_source": "of measured hbm_gbs" if measured_peaks() else "of fallback",
            "bytes": "N*K + 4N + 2MK + 2MN per call", "points": points,
            "best_GB/s": best["GB/s"], "best_frac": best["frac"],
            "worst_GB/s": worst["GB/s"], "worst_frac": worst["frac"]}


def measure_quant(i8, torch, dev, st, world, dist, reps: int = 40):
    """The fused quantiser alone on the Llama-7B prefill activation shapes (4096 tokens x 4096
    and x 11008 features).  Launched with threshold 0, i8_quantize_rowwise is exactly one
    quantiser kernel; with threshold 6 it adds the bitmap memset and the column-zeroing kernel.
    Inputs rotate over enough copies (> 2 x L2) that every call reads X from HBM.
    Algorithmic bytes per call: 2MK (X) + MK (codes) + 4M (scales) + K/8 (bitmap)."""
    hbm = (measured_peaks() or {}).get("hbm_gbs", 6650.0)
    res = []
    for M, K in ((4096, 4096), (4096, 11008)):
        X, _ = wl.activation(wl.BASE_SEED + 900 + K, M, K, round(0.001 * K), (20.0, 60.0))
        per = 3 * M * K
        n = max(4, int(np.ceil(2.5 * 126e6 / per)))
        Xs = [torch.from_numpy(X).to(dev) for _ in range(n)]
        CAs = [torch.empty((M, K), dtype=torch.int8, device=dev) for _ in range(n)]
        SCA = torch.empty((M,), dtype=torch.float32, device=dev)
        bm = torch.empty(((K + 31) // 32,), dtype=torch.int32, device=dev)
        row = {"shape": f"{M}x{K}"}
        for tau in (0.0, 6.0):
            for i in range(n):
                i8.i8_quantize_rowwise(Xs[i], tau, CA=CAs[i], SCA=SCA, bitmap=bm)
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize(dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(st)
            for r in range(reps):
                i8.i8_quantize_rowwise(Xs[r % n], tau, CA=CAs[r % n], SCA=SCA, bitmap=bm)
            e1.record(st)
            torch.cuda.synchronize(dev)
            us = e0.elapsed_time(e1) / reps * 1e3
            byts = 2 * M * K + M * K + 4 * M + K / 8
            gbs = byts / us / 1e3
            if tau == 0.0:
                # the kernel alone: the calls replayed from a graph (an eager call's host side
                # takes longer than this kernel)
                order = iter(range(reps))

                def one():  # the next input of the rotation
                    r = next(order)
                    i8.i8_quantize_rowwise(Xs[r % n], tau, CA=CAs[r % n], SCA=SCA, bitmap=bm)
                ug = graph_us(torch, dev, st, one, reps)
                row.update({"kernel_us": round(ug, 2), "kernel_GB/s": round(byts / ug / 1e3, 1),
                            "kernel_frac": round(byts / ug / 1e3 / hbm, 4),
                            "eager_us": round(us, 2), "eager_frac": round(gbs / hbm, 4)})
            else:
                row.update({"op_tau6_us": round(us, 2), "op_tau6_GB/s": round(gbs, 1),
                            "op_tau6_frac": round(gbs / hbm, 4)})
        res.append(row)
        del Xs, CAs
    return {"kernel": "k_quant_rows", "peak_gbs": hbm,
            "peak_source": "of measured hbm_gbs" if measured_peaks() else "of fallback",
            "bytes": "2MK + MK + 4M + K/8 per call",
            "timing": f"CUDA events over {reps} calls, inputs rotated over > 2 x L2; kernel_us: threshold 0, "
                      "the quantiser kernel alone, the calls replayed from one CUDA graph; eager_us: the same "
                      "calls issued from Python (host-bound); op_tau6_us: eager memset + quantiser + column "
                      "zeroing",
            "points": res}


def measure_nf4(i8, torch, dev, st, world, dist, reps: int = 20):
    """The 4-bit NF4 weight-only decode product on the Llama-70B FFN shapes at 1, 4 and 8 tokens:
    the packed weight (N*K/2 bytes) and its block scales (N*K/16 bytes) stream from HBM every call
    (117 MB + 15 MB, > L2).  Weights quantised once on the GPU (load time)."""
    hbm = (measured_peaks() or {}).get("hbm_gbs", 6650.0)
    points = []
    for N, K in ((28672, 8192), (8192, 28672)):
        packed, absmax = i8.i8_nf4_quantize(torch.from_numpy(wl.weight(950 + N, N, K)).to(dev))
        for M in (1, 4, 8):
            X, _ = wl.activation(wl.BASE_SEED + 951 + M, M, K, 8, (30.0, 30.0))
            dX = torch.from_numpy(X).to(dev)
            out = torch.empty((M, N), dtype=torch.float16, device=dev)
            for _ in range(3):
                i8.i8_nf4_gemv(dX, packed, absmax, out=out)
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize(dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(st)
            for _ in range(reps):
                i8.i8_nf4_gemv(dX, packed, absmax, out=out)
            e1.record(st)
            torch.cuda.synchronize(dev)
            us = e0.elapsed_time(e1) / reps * 1e3
            byts = N * K // 2 + N * (K // 64) * 4 + 2 * M * K + 2 * M * N
            gbs = byts / us / 1e3
            points.append({"shape": f"{M}x{K}->{N}", "tokens": M, "us": round(us, 2), "GB/s": round(gbs, 1),
                           "frac": round(gbs / hbm, 4)})
        del packed, absmax
    return {"kernel": "k_nf4_gemv", "peak_gbs": hbm,
            "peak_source": "of measured hbm_gbs" if measured_peaks() else "of fallback",
            "bytes": "N*K/2 + 4*N*K/64 + 2MK + 2MN per call", "points": points}


def cpu_per_config(layers_by_key, rows: int, min_seconds: float):
    """The oracle on a bounded row sample of each other workload family, one timing each."""
    res = {}
    for key, (layers_np, byts) in layers_by_key.items():
        times, ops = cpu_oracle_steps(layers_np, rows, 1, min_seconds=min_seconds)
        t = sum(times) / len(times)
        n_rows = [min(rows, X.shape[0]) for X, *_ in layers_np]
        e = {"TOPS": ops / t / 1e12, "sample_rows": n_rows, "passes": len(times), "s_per_pass": t}
        if byts is not None:
            e["GB/s"] = byts / t / 1e9
        res[key] = e
    return res


def measure_backward(i8, torch, dev, st, world, dist, reps: int = 20):
    """Input gradient through the frozen int8 layer for the distinct weight shapes of the
    Llama-7B-shaped layer at 4096 tokens: the transposed dequantisation of the weight
    (HBM-bound, 3NK bytes) and dX = dY . W^ on the fp16 tensor cores (2MNK flops), each
    timed alone with CUDA events over `reps` back-to-back calls (the dequantisation, shorter
    than its host call, from a CUDA graph of `reps` calls; dequant_t_eager_us issued from Python)."""
    layers = wl.workloads()["C3"].layers
    peaks = measured_peaks()
    f16_peak = float(peaks["bf16_tflops"]) if peaks else 1590.0
    hbm = float(peaks["hbm_gbs"]) if peaks else 6650.0
    points, seen = [], set()

    def timed(fn):
        for _ in range(3):
            fn()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        for _ in range(reps):
            fn()
        e1.record(st)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / reps * 1e3  # us per call

    for li, L in enumerate(layers):
        if (L.N, L.K) in seen:
            continue
        seen.add((L.N, L.K))
        CB, SCB, _ = i8.i8_quantize_rowwise(torch.from_numpy(wl.weight(500 + li, L.N, L.K)).to(dev), 0.0)
        dY = torch.from_numpy(wl.grad_output(600 + li, L.M, L.N)).to(dev)
        Wt = torch.empty((L.K, L.N), dtype=torch.float16, device=dev)
        dX = torch.empty((L.M, L.K), dtype=torch.float16, device=dev)
        us_dq_eager = timed(lambda: i8.i8_dequant_transposed(CB, SCB, Wt))
        us_dq = graph_us(torch, dev, st, lambda: i8.i8_dequant_transposed(CB, SCB, Wt), reps)
        us_mm = timed(lambda: i8.i8_linear8bit_backward_input(dY, Wt, dX))
        gbs = 3.0 * L.N * L.K / us_dq / 1e3
        tflops = 2.0 * L.M * L.N * L.K / us_mm / 1e6
        points.append({"layer": L.name, "dY": f"{L.M}x{L.N}", "W": f"{L.N}x{L.K}",
                       "dequant_t_us": round(us_dq, 2), "dequant_t_GB/s": round(gbs, 1),
                       "dequant_t_frac": round(gbs / hbm, 4), "dequant_t_eager_us": round(us_dq_eager, 2),
                       "gemm_us": round(us_mm, 2), "gemm_TFLOP/s": round(tflops, 1),
                       "gemm_frac": round(tflops / f16_peak, 4)})
    return {"metric": "input-gradient fp16 GEMM TFLOP/s (2MNK/s) and transposed dequant GB/s",
            "gemm_peak_tflops": f16_peak, "hbm_peak_gbs": hbm,
            "peak_source": ("of measured: fp16 = bf16_tflops (nominal fp16:bf16 = 1:1), hbm_gbs" if peaks
                            else "of fallback: 1.59 PFLOP/s, 6.65 TB/s"),
            "points": points}


GRAPH_CALLS = 20


def measure_other(i8, torch, dev, st, world, dist, reps: int = 50):
    """The other workload families, each forward timed alone with CUDA events over `reps`
    back-to-back calls (3 warm-up calls first):
      - the single 16x1024 -> 1024 linear, launch-latency bound: eager (back-to-back calls
        from Python), one call captured in a CUDA graph and replayed, and GRAPH_CALLS calls
        captured in one graph (time per forward);
      - the OPT-350m-shaped MLP pair at 512 tokens (fc2 fed the ReLU of the GPU's fc1 output,
        computed before timing);
      - the Llama-13B MLP shape 2048x5120 -> 13824 over outlier fractions {0, 0.1, 1, 5} %
        and thresholds {0, 6} (one weight for all points), which exercises the many-outlier
        tcgen05 fp16 path above 16 columns."""
    W = wl.workloads()
    peaks = measured_peaks()
    peak = 2.0 * float(peaks["bf16_tflops"]) if peaks else 3180.0

    def run(L, dX, CB, SCB, db, out, ws):
        i8.i8_linear8bit_forward(dX, CB, SCB, db, L.threshold, out=out, workspace=ws,
                                 max_outlier_cols=MAX_OUTLIER_COLS)

    def timed(fn, n=reps):
        for _ in range(3):
            fn()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        for _ in range(n):
            fn()
        e1.record(st)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / n * 1e3

    def prepared(key, li, L, X=None, weight=None):
        Xh, _, Wh, b = wl.layer_inputs(wl.seed_of(key), li, L)
        if weight is None:
            CB, SCB, _ = i8.i8_quantize_rowwise(torch.from_numpy(Wh).to(dev), 0.0)
        else:
            CB, SCB = weight
        dX = X if X is not None else torch.from_numpy(Xh).to(dev)
        db = None if b is None else torch.from_numpy(b).to(dev)
        out = torch.empty((L.M, L.N), dtype=torch.float16, device=dev)
        ws = torch.empty((i8.i8_linear8bit_workspace_size(L.M, L.N, L.K, MAX_OUTLIER_COLS),),
                         dtype=torch.uint8, device=dev)
        return dX, CB, SCB, db, out, ws

    def status(ws):
        code, count = i8.i8_read_status(ws)
        if code != 0:
            raise RuntimeError(f"device status {i8.STATUS.get(code, code)}")
        return count

    res = {"peak_tops": peak, "peak_source": ("of measured: int8 = 2 x bf16_tflops" if peaks
                                              else "of fallback: int8 = 2 x 1.59 PFLOP/s")}
    # single linear: eager and graph-replayed
    L = W["C1"].layers[0]
    a = prepared("C1", 0, L)
    dX, CB, SCB, db, out, _ = a
    layer = i8.Linear8bitLt(CB, SCB, db, L.threshold, MAX_OUTLIER_COLS)
    us_eager_fn = timed(lambda: run(L, *a))
    us_eager = timed(lambda: layer(dX, out=out))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        layer(dX, out=out)
    us_graph_1 = timed(graph.replay)
    del graph
    # a graph of GRAPH_CALLS forwards: the device time per forward once the host no longer
    # issues each launch (one replay of a one-forward graph is bound by the host call)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(GRAPH_CALLS):
            layer(dX, out=out)
    us_graph = timed(graph.replay, n=max(1, reps // 5)) / GRAPH_CALLS
    del graph
    res["single_linear"] = {"shape": f"{L.M}x{L.K}->{L.N}", "outlier_cols": status(layer.last_workspace),
                            "us_eager": round(us_eager, 2), "us_graph": round(us_graph, 2),
                            "api": "Linear8bitLt layer (weights checked once); "
                                   "us_eager_function: i8_linear8bit_forward with every argument checked",
                            "us_eager_function": round(us_eager_fn, 2),
                            "us_graph_one_per_replay": round(us_graph_1, 2),
                            "graph_calls": GRAPH_CALLS,
                            "TOPS_eager": round(L.ops / us_eager / 1e6, 2),
                            "TOPS_graph": round(L.ops / us_graph / 1e6, 2)}
    # OPT-350m MLP pair
    fc1, fc2 = W["C2"].layers
    a1 = prepared("C2", 0, fc1)
    run(fc1, *a1)
    x2 = torch.relu(a1[4]).contiguous()
    a2 = prepared("C2", 1, fc2, X=x2)
    us1 = timed(lambda: run(fc1, *a1))
    us2 = timed(lambda: run(fc2, *a2))
    res["opt350m_mlp"] = {"fc1": {"shape": f"{fc1.M}x{fc1.K}->{fc1.N}", "outlier_cols": status(a1[5]),
                                  "us": round(us1, 2), "TOPS": round(fc1.ops / us1 / 1e6, 1)},
                          "fc2": {"shape": f"{fc2.M}x{fc2.K}->{fc2.N}", "outlier_cols": status(a2[5]),
                                  "us": round(us2, 2), "TOPS": round(fc2.ops / us2 / 1e6, 1)}}
    # Llama-13B MLP outlier sweep
    keys = [k for k in W if k.startswith("C5_")]
    weight = None
    points = []
    for key in keys:
        L = W[key].layers[0]
        if weight is None:
            _, _, Wh, _ = wl.layer_inputs(wl.seed_of(keys[0]), 0, L)
            CB, SCB, _ = i8.i8_quantize_rowwise(torch.from_numpy(Wh).to(dev), 0.0)
            weight = (CB, SCB)
        a = prepared(key, 0, L, weight=weight)
        us = timed(lambda: run(L, *a), n=20)
        tops = L.ops / us / 1e6
        n_cols = status(a[5])
        # the two halves of the same forward, each timed alone: quantise + outlier preparation,
        # then the GEMM with its epilogue (it re-reads the prepared workspace)
        dX, CB, SCB, db, out, ws = a
        def prep():
            i8.i8_linear8bit_prepare(dX, CB, L.threshold, ws, MAX_OUTLIER_COLS)

        def gemm():
            i8.i8_linear8bit_matmul_dequant(CB, SCB, db, L.M, L.threshold, out, ws, MAX_OUTLIER_COLS)
        timed(prep, n=3)
        us_prep = graph_us(torch, dev, st, prep, 20)
        timed(gemm, n=3)
        us_gemm = graph_us(torch, dev, st, gemm, 20)
        status(ws)
        points.append({"key": key, "threshold": L.threshold, "planted_cols": L.n_out,
                       "outlier_cols": n_cols, "us": round(us, 2), "TOPS": round(tops, 1),
                       "frac": round(tops / peak, 4), "prepare_us": round(us_prep, 2),
                       "gemm_us": round(us_gemm, 2)})
    res["llama13b_mlp_sweep"] = {"shape": "2048x5120->13824", "points": points,
                                 "split": "prepare_us / gemm_us: the forward's two halves, each timed alone "
                                          "(20 calls replayed from a CUDA graph)"}
    return res


def measure_shared_inputs(i8, torch, dev, st, world, dist, layers, reps: int = 20):
    """The headline's seven linears fed the way a decoder layer feeds them: q/k/v read one X
    and gate/up read one X, so each of those groups is one i8_linear8bit_forward_multi call
    (X quantised and its outlier columns found once); o and down stay single forwards.  Same
    weights, shapes and ops as the headline step; the inputs of k, v and up are q's and
    gate's."""
    by = {d["L"].name: d for d in layers}
    groups = [["q_proj", "k_proj", "v_proj"], ["o_proj"], ["gate_proj", "up_proj"], ["down_proj"]]
    if any(n not in by for g in groups for n in g) or len(layers) != 7:
        return None
    plan, launches = [], 0
    for names in groups:
        ds = [by[n] for n in names]
        L0 = ds[0]["L"]
        ws = None
        if len(ds) > 1:
            ws = torch.empty((i8.i8_linear8bit_multi_workspace_size(L0.M, L0.K, [d["L"].N for d in ds],
                                                                    MAX_OUTLIER_COLS),), dtype=torch.uint8, device=dev)
        plan.append((ds, ws))
        launches += 3 + 2 * (len(ds) - 1)   # quantise, prepare, GEMM; per further weight: gather + GEMM

    def step():
        for ds, ws in plan:
            L0 = ds[0]["L"]
            if ws is None:
                d = ds[0]
                i8.i8_linear8bit_forward(d["X"], d["CB"], d["SCB"], d["b"], L0.threshold, out=d["out"],
                                         workspace=d["ws"], max_outlier_cols=MAX_OUTLIER_COLS)
            else:
                i8.i8_linear8bit_forward_multi(ds[0]["X"], [d["CB"] for d in ds], [d["SCB"] for d in ds],
                                               [d["b"] for d in ds], L0.threshold, outs=[d["out"] for d in ds],
                                               workspace=ws, max_outlier_cols=MAX_OUTLIER_COLS)

    for _ in range(3):
        step()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(reps):
        step()
    e1.record(st)
    torch.cuda.synchronize(dev)
    for ds, ws in plan:
        code, _ = i8.i8_read_status(ws if ws is not None else ds[0]["ws"])
        if code != 0:
            raise RuntimeError(f"device status {i8.STATUS.get(code, code)}")
    ms = e0.elapsed_time(e1) / reps
    ops = sum(d["L"].ops for d in layers)
    return {"metric": "TOPS (2MNK/s) of the same seven linears with q/k/v and gate/up sharing their input",
            "ms_per_step": ms, "TOPS": ops / ms / 1e9, "steps": reps, "gpu_launches_per_step": launches,
            "calls": "forward_multi(q,k,v) + forward(o) + forward_multi(gate,up) + forward(down)"}


def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:  # noqa: BLE001
        pass
    return os.cpu_count() or 1


def oracle_layers(W: wl.Workload, seed: int, weight_rows=None):
    """Oracle operands of every linear of a workload.  `weight_rows` keeps only the first
    rows of each weight (a sample of the output columns; the outlier set and row scales
    still come from the whole of X)."""
    import oracle
    out = []
    for li, L in enumerate(W.layers):
        X, _, Wt, b = wl.layer_inputs(seed, li, L)
        if X is None:   # chained input: the oracle feeds itself (ReLU of its own previous output)
            pX, pCB, pSCB, pb, ptau = out[-1]
            X = np.maximum(oracle.linear8bit_forward(pX, pCB, pSCB, pb, ptau), np.float16(0))
        if weight_rows is not None:
            Wt = Wt[:weight_rows]
            b = None if b is None else b[:weight_rows]
        CB, SCB = oracle.quantize_weight_rowwise(Wt)
        out.append((X, CB, SCB, b, L.threshold))
    return out


# ------------------------------------------------------------------ reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    W = wl.workloads()[args.workload]
    layers_np = oracle_layers(W, wl.seed_of(args.workload))
    rows = args.cpu_rows
    cpu_oracle_steps(layers_np, rows, max(args.warmup, 0))
    times, ops = cpu_oracle_steps(layers_np, rows, args.steps)
    t = sum(times)
    value = ops * args.steps / t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": {"workload": describe(W), "sample_rows_per_linear": rows, "parallelism": "replicas"},
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": cpu_threads(), "kind": "oracle",
                         "sample": f"first {rows} rows of every linear of the workload per step "
                                   "(oracle quantises the sample, exact int product, float64 dequant)"},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ our arm
def run_ours(args):
    import torch
    import torch.distributed as dist
    import int8_mixed_precision_vectorwise_b200 as i8
    from int8_mixed_precision_vectorwise_b200 import build

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device: the library has no CPU path")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    i8.lib()

    W = wl.workloads()[args.workload]
    seed = wl.seed_of(args.workload)
    st = torch.cuda.current_stream(dev)

    # ---- inputs (seeded host arrays -> HBM), weight prep on the GPU (load time)
    layers = []
    for li, L in enumerate(W.layers):
        X, _, Wt, b = wl.layer_inputs(seed, li, L)
        dW = torch.from_numpy(Wt).to(dev)
        CB, SCB, _ = i8.i8_quantize_rowwise(dW, 0.0)
        del dW
        dX = torch.from_numpy(X).to(dev) if X is not None else None
        db = torch.from_numpy(b).to(dev) if b is not None else None
        out = torch.empty((L.M, L.N), dtype=torch.float16, device=dev)
        ws = torch.empty((i8.i8_linear8bit_workspace_size(L.M, L.N, L.K, MAX_OUTLIER_COLS),),
                         dtype=torch.uint8, device=dev)
        layers.append(dict(L=L, X=dX, CB=CB, SCB=SCB, b=db, out=out, ws=ws, X_host=X))
    for li, d in enumerate(layers):      # chained inputs read the previous layer's output buffer
        if d["X"] is None:
            d["X"] = layers[li - 1]["out"]
            d["chained"] = True
    ops_per_step = sum(d["L"].ops for d in layers)
    n_launch_per_step = sum(2 + (1 if d["L"].threshold > 0 else 0) for d in layers)

    def step(gemm_events=None):
        for li, d in enumerate(layers):
            L = d["L"]
            i8.i8_linear8bit_prepare(d["X"], d["CB"], L.threshold, d["ws"], MAX_OUTLIER_COLS)
            if gemm_events is not None:
                gemm_events[li][0].record(st)
            i8.i8_linear8bit_matmul_dequant(d["CB"], d["SCB"], d["b"], L.M, L.threshold, d["out"], d["ws"],
                                            MAX_OUTLIER_COLS)
            if gemm_events is not None:
                gemm_events[li][1].record(st)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(max(args.warmup, 3)):
        step()
    for d in layers:
        code, _ = i8.i8_read_status(d["ws"])
        if code != 0:
            raise RuntimeError(f"device status {i8.STATUS.get(code, code)} on {d['L'].name}")

    K = args.steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev)
    barrier()
    with sampler:
        # headline: K bare steps (no events between kernels, which would stop each
        # kernel from being scheduled while its predecessor finishes)
        e0.record(st)
        for k in range(K):
            step()
        e1.record(st)
        barrier()
        # roofline: the same K steps again with an event pair around every GEMM
        ev = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)] for _ in layers]
              for _ in range(K)]
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(st)
        for k in range(K):
            step(ev[k])
        g1.record(st)
        barrier()
    ms = e0.elapsed_time(e1)
    ms_instr = g0.elapsed_time(g1)
    gemm_step_ms = [sum(a.elapsed_time(b) for a, b in row) for row in ev]
    gemm_ms = sum(gemm_step_ms)
    ms_max = max_over_ranks(ms, world, dist, dev)

    # ---- the same step with the inputs shared as in a decoder layer (informational)
    shared = None
    if not args.no_shared and args.workload == "C3":
        shared = measure_shared_inputs(i8, torch, dev, st, world, dist, layers)

    # ---- end to end: host inputs -> device -> forward -> host outputs, per step
    e2e = None
    if not args.no_e2e:
        h_in = []
        for d in layers:
            h_in.append(None if d.get("chained") else torch.from_numpy(d["X_host"]).pin_memory())
        h_out = [torch.empty(d["out"].shape, dtype=torch.float16).pin_memory() for d in layers]
        Ke = min(K, 20)
        # Copies run on their own streams so that the host-to-device copy of the
        # next linear's input and the device-to-host copy of the previous
        # output (the two directions of the link) overlap the forward: the
        # forward of linear i waits for its input; the copy of an output waits
        # for its forward; a forward that rewrites `out` waits for the copy of
        # its previous contents; a copy that rewrites `X` waits for the forward
        # that read its previous contents.
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in layers]
        ev_fwd = [torch.cuda.Event() for _ in layers]
        ev_out = [torch.cuda.Event() for _ in layers]
        started = [False] * len(layers)

        def e2e_step():
            for li, d in enumerate(layers):
                L = d["L"]
                if h_in[li] is not None:
                    with torch.cuda.stream(s_in):
                        if started[li]:
                            s_in.wait_event(ev_fwd[li])
                        d["X"].copy_(h_in[li], non_blocking=True)
                        ev_in[li].record(s_in)
                    st.wait_event(ev_in[li])
                if started[li]:
                    st.wait_event(ev_out[li])
                i8.i8_linear8bit_forward(d["X"], d["CB"], d["SCB"], d["b"], L.threshold, out=d["out"],
                                         workspace=d["ws"], max_outlier_cols=MAX_OUTLIER_COLS)
                ev_fwd[li].record(st)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_fwd[li])
                    h_out[li].copy_(d["out"], non_blocking=True)
                    ev_out[li].record(s_out)
                started[li] = True

        def join():
            for li in range(len(layers)):
                st.wait_event(ev_out[li])
        e2e_step()
        join()
        barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(st)
        for _ in range(Ke):
            e2e_step()
        join()
        f1.record(st)
        barrier()
        te = max_over_ranks(f0.elapsed_time(f1), world, dist, dev)
        h2d = sum(h.numel() * 2 for h in h_in if h is not None)
        d2h = sum(h.numel() * 2 for h in h_out)
        e2e = {"value": job_throughput(ops_per_step, Ke, world, te), "unit": "TOPS",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": Ke,
               "ms_per_step": te / Ke}

    for d in layers:
        code, _ = i8.i8_read_status(d["ws"])
        if code != 0:
            raise RuntimeError(f"device status {i8.STATUS.get(code, code)} on {d['L'].name}")

    # ---- decode regime (weight streaming): Llama-70B FFN shapes, few tokens
    decode = None
    if not args.no_decode:
        decode = measure_decode(i8, torch, dev, st, world, dist)

    # ---- input gradient (training through the frozen int8 layer)
    backward = None
    if not args.no_backward:
        backward = measure_backward(i8, torch, dev, st, world, dist)

    # ---- the other workload families (single linear, OPT MLP, outlier sweep)
    other_wl = None
    if not args.no_other:
        other_wl = measure_other(i8, torch, dev, st, world, dist)

    # ---- the quantiser alone (HBM roofline)
    quant = None
    if not args.no_quant:
        quant = measure_quant(i8, torch, dev, st, world, dist)

    # ---- the NF4 weight-only decode product (HBM roofline)
    nf4 = None
    if not args.no_nf4:
        nf4 = measure_nf4(i8, torch, dev, st, world, dist)

    # ---- CPU oracle baseline (rank 0, one GPU only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        layers_np = oracle_layers(W, seed)
        times, cops = cpu_oracle_steps(layers_np, args.cpu_rows, 3, min_seconds=10.0)
        cpu = {"value": cops * len(times) / sum(times) / 1e12, "unit": "TOPS", "cores": cpu_threads(),
               "kind": "oracle",
               "sample": f"first {args.cpu_rows} rows of each of the {len(layers_np)} linears, "
                         f"{len(times)} passes ({sum(times):.1f} s)"}
        # the other workload families, each on a bounded sample (first 64 activation rows; the
        # decode point on its 16 tokens and the first 2048 rows of each weight, bytes counted
        # for that sample)
        Wall = wl.workloads()
        dec = Wall["C4_t16_o8"]
        dec_np = oracle_layers(dec, wl.seed_of("C4_t16_o8"), weight_rows=2048)
        dec_bytes = sum(CB.shape[0] * CB.shape[1] + 4 * CB.shape[0] + 2 * X.shape[0] * X.shape[1]
                        + 2 * X.shape[0] * CB.shape[0] for X, CB, *_ in dec_np)
        per = {
            "C1_single_linear": (oracle_layers(Wall["C1"], wl.seed_of("C1")), None),
            "C2_opt350m_mlp": (oracle_layers(Wall["C2"], wl.seed_of("C2")), None),
            "C4_llama70b_decode_t16_o8": (dec_np, dec_bytes),
            "C5_llama13b_mlp_f0.01_t6": (oracle_layers(Wall["C5_f0.01_t6"], wl.seed_of("C5_f0.01_t6")), None),
        }
        cpu["per_config"] = cpu_per_config(per, 64, min_seconds=1.5)
        cpu["per_config_sample"] = ("first 64 activation rows of every linear (C1: all 16; C4: its 16 tokens "
                                    "and the first 2048 rows of each weight), repeated for >= 1.5 s")

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    clocks = sampler.summary()
    peaks = measured_peaks()
    # burst peak when the timed region ran at full clock (short region, no
    # power capping seen), the sustained one otherwise
    at_max = (clocks.get("sm_mhz") is not None and clocks.get("sm_max_mhz")
              and clocks["sm_mhz"] >= 0.97 * clocks["sm_max_mhz"])
    if peaks:
        key = "bf16_tflops" if at_max else "bf16_tflops_sustained"
        peak = 2.0 * float(peaks[key])
        peak_src = f"of measured: int8 = 2 x {key} (nominal int8:bf16 = 4.5:2.25)"
        other = 2.0 * float(peaks["bf16_tflops_sustained" if at_max else "bf16_tflops"])
    else:
        peak = 2.0 * (1590.0 if at_max else 1400.0)
        peak_src = "of fallback: int8 = 2 x " + ("1.59" if at_max else "1.4") + " PFLOP/s bf16"
        other = 2.0 * (1400.0 if at_max else 1590.0)
    gemm_launches = K * len(layers)
    achieved = ops_per_step * K / (gemm_ms / 1e3) / 1e12
    line = {
        "metric": METRIC,
        "value": job_throughput(ops_per_step, K, world, ms_max),
        "unit": "TOPS",
        "n_gpus": world,
        "steps": K,
        "warmup": max(args.warmup, 3),
        "ms_per_step": ms_max / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int8",
        "data": "synthetic",
        "config": {"workload": describe(W), "tokens": W.layers[0].M, "linears": len(layers),
                   "max_outlier_cols": MAX_OUTLIER_COLS,
                   "l2": "per-step working set > 126 MB L2 (int8 weights alone "
                         f"{sum(d['L'].N * d['L'].K for d in layers) / 1e6:.0f} MB); no flush",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "tensor", "kernel": "k_gemm_i8_tcgen05", "achieved": achieved, "peak": peak,
                     "unit": "TOPS", "frac": achieved / peak, "traffic": read_traffic(),
                     "peak_source": peak_src, "frac_of_other_peak": achieved / other,
                     "gemm_ms_per_step": gemm_ms / K, "gemm_share_of_step": gemm_ms / ms_instr,
                     "gemm_ms_per_step_p10_p50_p90": nearest_rank(gemm_step_ms, (0.1, 0.5, 0.9)),
                     "gemm_timing": "CUDA events around each GEMM launch in a second pass of the same "
                                    f"{K} steps ({ms_instr / K:.4f} ms per instrumented step)",
                     "quant": None if quant is None else {
                         "kernel": quant["kernel"], "bytes": quant["bytes"], "peak_gbs": quant["peak_gbs"],
                         "points": [[q["shape"], q["kernel_us"], q["kernel_GB/s"], q["kernel_frac"], q["eager_us"]]
                                    for q in quant["points"]],
                         "columns": ["shape", "us (graph)", "GB/s", "frac", "us (eager)"]},
                     "decode": None if decode is None else {
                         "kernel": "k_decode_prep + k_gemm_i8_decode (whole forward)", "bytes": decode["bytes"],
                         "peak_gbs": decode["peak_gbs"],
                         "points": [[q["tokens"], q["outlier_cols"], q["shape"], q["us"], q["GB/s"], q["frac"],
                                     q["us_graph"], q["frac_graph"]] for q in decode["points"]],
                         "columns": ["tokens", "outlier_cols", "shape", "us", "GB/s", "frac", "us (graph)",
                                     "frac (graph)"]},
                     "nf4": None if nf4 is None else {
                         "kernel": nf4["kernel"], "bytes": nf4["bytes"], "peak_gbs": nf4["peak_gbs"],
                         "points": [[q["shape"], q["us"], q["GB/s"], q["frac"]] for q in nf4["points"]],
                         "columns": ["shape", "us", "GB/s", "frac"]}},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "decode": decode,
        "quant": quant,
        "nf4": nf4,
        "backward": backward,
        "other_workloads": other_wl,
        "shared_inputs": shared,
        "clocks": clocks,
        "gpu_launches": K * n_launch_per_step,
        "gpu_launches_note": f"per step per linear: quantise + outlier prepare + GEMM ({gemm_launches} GEMMs)",
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
