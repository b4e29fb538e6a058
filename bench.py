#!/usr/bin/env python
"""Benchmark of the fused attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one attention forward (every step of the hot path: tile schedule, Q/K/V TMA
loads, Q K^T and P V on the tensor cores, online softmax, epilogue; plus the tile-map build
for document masks) over one batch of the named workload, inputs already in HBM.  Prints
one JSON line.  With N > 1 (launched by torchrun) every rank runs its own copy of the
workload (independent (b, h) units, no collective on the data path): weak scaling, value =
all ranks' FLOPs / the slowest rank's device time.

``--impl reference`` times the fp64 CPU oracle instead (rank 0 only), on a bounded sample
of the same workload, with the same metric and unit.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from attn_workloads import (MASK_CAUSAL, MASK_DOC, MASK_WINDOW, WORKLOADS, alibi_slopes,  # noqa: E402
                            doc_lengths, make_doc_ids, make_fp8_source, make_qkv, varlen_cu_seqlens)

METRIC = "attention fwd TFLOP/s and % of B200 dense BF16/FP8 tensor peak, per config"
L2_BYTES = 126 * 1024 * 1024


# ----------------------------------------------------------------------------- FLOP counts
def visible_pairs(w) -> int:
    """Exact number of visible (i, j) pairs over the whole batch (all b, h)."""
    Sq, Sk = w.Sq, w.Sk
    d = Sk - Sq
    if w.mask_kind & MASK_DOC or w.varlen:
        per_b = []
        for b in range(w.B):
            lens = doc_lengths(Sq, b)
            if w.mask_kind & MASK_CAUSAL:
                per_b.append(sum(n * (n + 1) // 2 for n in lens))
            else:
                per_b.append(sum(n * n for n in lens))
        return sum(per_b) * w.H
    total = 0
    i = np.arange(Sq, dtype=np.int64)
    ip = i + d
    hi = np.full(Sq, Sk - 1, dtype=np.int64)
    lo = np.zeros(Sq, dtype=np.int64)
    if w.mask_kind & MASK_CAUSAL:
        hi = np.minimum(hi, ip)
    if w.mask_kind & MASK_WINDOW:
        lo = np.maximum(lo, ip - w.window + 1)
        if not (w.mask_kind & MASK_CAUSAL):
            hi = np.minimum(hi, ip + w.window - 1)
    total = int(np.clip(hi - lo + 1, 0, None).sum())
    return total * w.B * w.H


def algorithmic_flops(w) -> float:
    """4 * D per visible pair (2 for Q K^T, 2 for P V)."""
    return 4.0 * w.D * visible_pairs(w)


def tile_count_flops(w) -> float:
    """FLOPs counted over the 256x128 tiles the kernel visits (analytic masks only)."""
    if w.mask_kind & MASK_DOC or w.varlen:
        return float("nan")
    nqb = (w.Sq + 255) // 256
    d = w.Sk - w.Sq
    tiles = 0
    for qb in range(nqb):
        A = qb * 256 + d
        Bm = min(qb * 256 + 255, w.Sq - 1) + d
        causal, win = w.mask_kind & MASK_CAUSAL, w.mask_kind & MASK_WINDOW
        if causal:
            A = max(A, 0)
        lo = max(0, A - w.window + 1) if win else 0
        hi = Bm if causal else (Bm + w.window - 1 if win else w.Sk - 1)
        hi = min(hi, w.Sk - 1)
        if (causal and Bm < 0) or hi < lo:
            continue
        tiles += hi // 128 - lo // 128 + 1
    return 4.0 * w.D * 256 * 128 * tiles * w.B * w.H


# ----------------------------------------------------------------------------- ranks
def max_over_ranks(x: float, dist=None, device="cpu") -> float:
    """Max of a per-rank time over all ranks (identity without a process group)."""
    if dist is None:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(flops_per_step: float, steps: int, world: int, ms: float) -> float:
    """Whole-job TFLOP/s: every rank ran `steps` steps of the same workload; `ms` is the
    slowest rank's device time."""
    return flops_per_step * steps * world / (ms * 1e-3) / 1e12


# ----------------------------------------------------------------------------- peaks, clocks
def measured_peaks():
    """Roofline denominators.  BF16 and HBM from MEASURED_PEAKS.json (written on this pool's
    B200s); FP8 e4m3 from profiles/fp8_peak.json (written by ``bench.py --measure-fp8-peak``
    on a B200), else the BF16 figure times the nominal dense FP8/BF16 ratio (4.5 / 2.25)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        out = {"bf16": d["bf16_tflops"], "bf16_sustained": d.get("bf16_tflops_sustained"),
               "hbm": d["hbm_gbs"], "source": "measured"}
    else:
        out = {"bf16": 1590.0, "bf16_sustained": 1400.0, "hbm": 6650.0, "source": "fallback"}
    f = os.path.join(ROOT, "profiles", "fp8_peak.json")
    if os.path.exists(f):
        d = json.load(open(f))
        out.update(fp8=d["fp8_tflops"], fp8_sustained=d.get("fp8_tflops_sustained"),
                   fp8_source="measured e4m3 GEMM (profiles/fp8_peak.json)")
    else:
        out.update(fp8=out["bf16"] * 2.0, fp8_sustained=(out["bf16_sustained"] or 0.0) * 2.0,
                   fp8_source="bf16 x 2 (nominal dense fp8/bf16 ratio)")
    # no FP4 GEMM is measured: the FP8 figure times the nominal dense FP4/FP8 ratio (9 / 4.5)
    out.update(fp4=out["fp8"] * 2.0, fp4_sustained=(out["fp8_sustained"] or 0.0) * 2.0,
               fp4_source=out["fp8_source"] + " x 2 (nominal dense fp4/fp8 ratio)")
    return out


def peak_key(w) -> str:
    return "fp4" if w.fp4 else ("fp8" if w.fp8 else "bf16")


def dtype_of(w) -> str:
    return "e2m1" if w.fp4 else ("e4m3" if w.fp8 else "bf16")


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index: int, period_s: float = 0.005):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], set()
        self._stop = threading.Event()
        self.max_mhz = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

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
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# The sources that make up each forward attention kernel family and its launch: BF16/FP8
# (attn_fwd_kernel) and FP4 (attn_fp4_kernel, which also uses the BF16 kernel's helpers).  The
# backward, quantiser and tile-map sources do not change them.
BF16_SOURCES = ("attn_fwd_kernel.cuh", "ptx.cuh", "tmem_moves.cuh", "attn_api.cu")
FP4_SOURCES = BF16_SOURCES + ("attn_fp4_kernel.cuh", "attn_fp4_api.inc")
FWD_SOURCES = FP4_SOURCES


def code_only(text: str) -> str:
    """The source without its comments and blank lines (no source here puts a comment marker
    inside a string literal), so that a comment edit does not invalidate a capture."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*", "", line).rstrip() for line in text.splitlines())
    return "\n".join(line for line in lines if line.strip())


def kernel_source_hash(family: str = "bf16") -> str:
    """Hash of the code (comments and blank lines removed) of one kernel family's sources."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "tiled_attention_14_b200", "csrc")
    for f in (FP4_SOURCES if family == "fp4" else BF16_SOURCES):
        h.update(code_only(open(os.path.join(csrc, f), encoding="utf-8").read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per launch of the attention kernel from the committed ncu summary, if the
    kernel source has not changed since it was captured."""
    p = os.path.join(ROOT, "profiles", f"traffic_{workload}.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    w = WORKLOADS.get(workload)
    if d.get("kernel_source_hash") != kernel_source_hash("fp4" if (w is not None and w.fp4) else "bf16"):
        return None
    return d.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------- CPU oracle leg
_FP4_INPUTS = {}


def oracle_sample_fp4(w, budget_s: float, seed: int = 0):
    """The FP4 oracle on evenly spaced query rows of one (b, h) head: the oracle's MXFP4
    quantisation of that head's Q, K, V (done once, not timed), then its Direct-P attention
    in fp64 (timed).  Returns (algorithmic FLOPs done, seconds, description)."""
    from oracle import fp4
    key = (w.name, w.Sq, w.Sk, seed)
    if key not in _FP4_INPUTS:
        q, k, v = (t.float().numpy() for t in make_qkv(1, 1, w.Sq, w.Sk, w.D, seed=seed))

        def deq(x):
            c, X = fp4.mx_quantize(x, axis=-1)
            return fp4.mx_dequantize(c, X, axis=-1)[..., :x.shape[-1]]
        vh = np.swapaxes(deq(np.swapaxes(v, -1, -2)), -1, -2)
        _FP4_INPUTS.clear()
        _FP4_INPUTS[key] = (deq(q), deq(k), vh)
    qh, kh, vh = _FP4_INPUTS[key]
    probe = np.arange(min(w.Sq, 64))
    t0 = time.perf_counter()
    fp4.attention_fp4_fwd(qh, kh, vh, w.scale, rows=probe)
    t_probe = time.perf_counter() - t0
    n = max(len(probe), min(w.Sq, int(len(probe) * budget_s / max(t_probe, 1e-6))))
    rows = np.linspace(0, w.Sq - 1, num=n).astype(np.int64)
    t0 = time.perf_counter()
    fp4.attention_fp4_fwd(qh, kh, vh, w.scale, rows=rows)
    dt = time.perf_counter() - t0
    return 4.0 * w.D * w.Sk * len(rows), dt, (f"{len(rows)} of {w.Sq} query rows (evenly spaced) of one (b,h) "
                                              f"head of the {w.note} workload (Direct-P oracle on the oracle's "
                                              f"MXFP4 inputs; quantisation not timed)")


def oracle_sample(w, budget_s: float, seed: int = 0):
    """Times the fp64 oracle on the workload until about budget_s of CPU work is done:
    whole (b, h) heads while one head fits the budget, else an evenly spaced subset of one
    head's query rows.  Returns (algorithmic FLOPs done, seconds, description)."""
    if w.fp4:
        return oracle_sample_fp4(w, budget_s, seed)
    from oracle.attention import attention_fwd, visible_mask
    q, k, v = make_qkv(1, 1, w.Sq, w.Sk, w.D, seed=seed)
    sl = alibi_slopes(w.H)[:1].numpy() if w.alibi else None
    # packed sequences of the document lengths attend exactly as the document mask does
    doc = make_doc_ids(1, w.Sq) if (w.doc or w.varlen) else None
    doc_np = None if doc is None else doc[0].numpy()
    if w.varlen:
        import dataclasses
        w = dataclasses.replace(w, mask_kind=w.mask_kind | MASK_DOC)

    def flops_of(rows):
        vis = 0
        for r0 in range(0, len(rows), 1024):
            vis += int(visible_mask(rows[r0:r0 + 1024], w.Sq, w.Sk, w.mask_kind, w.window, doc_np).sum())
        return 4.0 * w.D * vis

    probe = np.arange(min(w.Sq, 256))
    t0 = time.perf_counter()
    attention_fwd(q, k, v, w.scale, w.mask_kind, w.window, w.softcap, sl, doc, rows=probe)
    t_probe = time.perf_counter() - t0
    est_head = t_probe * w.Sq / len(probe)
    if est_head > budget_s:
        n = max(len(probe), int(len(probe) * budget_s / max(t_probe, 1e-6)))
        rows = np.linspace(0, w.Sq - 1, num=min(n, w.Sq)).astype(np.int64)
        t0 = time.perf_counter()
        attention_fwd(q, k, v, w.scale, w.mask_kind, w.window, w.softcap, sl, doc, rows=rows)
        dt = time.perf_counter() - t0
        return flops_of(rows), dt, (f"{len(rows)} of {w.Sq} query rows (evenly spaced) of one (b,h) "
                                    f"head of the {w.note} workload")
    rows = np.arange(w.Sq)
    per_head = flops_of(rows)
    heads, dt = 0, 0.0
    while heads < w.B * w.H and (heads == 0 or dt < budget_s):
        t0 = time.perf_counter()
        attention_fwd(q, k, v, w.scale, w.mask_kind, w.window, w.softcap, sl, doc)
        dt += time.perf_counter() - t0
        heads += 1
    return per_head * heads, dt, (f"{heads} of {w.B * w.H} whole (b,h) heads of the {w.note} workload "
                                  f"(all {w.Sq} query rows each)")


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    budget = min(15.0, max(1.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(w, budget * 0.2)
    vals, times = [], []
    desc = ""
    for _ in range(args.steps):
        f, dt, desc = oracle_sample(w, budget)
        vals.append(f / dt / 1e12)
        times.append(dt)
    value = float(np.mean(vals))
    cores = blas_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": float(np.mean(times) * 1e3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config(w):
    return {"workload": w.note, "B": w.B, "H": w.H, "Hkv": w.kv_heads, "Sq": w.Sq, "Sk": w.Sk, "D": w.D,
            "packed_sequences": w.varlen,
            "mask": {"causal": bool(w.mask_kind & MASK_CAUSAL), "window": w.window,
                     "alibi": w.alibi, "softcap": w.softcap, "document": w.doc},
            "flops": "exact: 4*D per visible (i,j) pair",
            "l2": f"inputs larger than L2 ({(compulsory_bytes(w) - w.B * w.H * w.Sq * (w.D * 2 + 4)) / 1e6:.0f} MB "
                  f"of {'MXFP4 ' if w.fp4 else ''}Q/K/V{' and scales' if (w.fp4 or w.fp8) else ''} + "
                  f"{w.B * w.H * w.Sq * w.D * 2 / 1e6:.0f} MB of O vs 126 MB L2); no flush"}


# ----------------------------------------------------------------------------- GPU leg
class Case:
    """One workload resident on the device: its inputs, outputs and a step() that runs the
    whole hot path once through the public API (tile map + attention for documents)."""

    def __init__(self, ta, w, dev, seed):
        self.w, self.ta, self.dev = w, ta, dev
        self.stream = torch.cuda.current_stream(dev)
        self.cu = None
        if w.fp8:
            self.host = make_fp8_source(w.B, w.H, w.Sq, w.D, seed=seed)
        elif w.varlen:
            # B batch rows of S tokens each, packed token-major [T, H, D]
            cu = varlen_cu_seqlens(w.B, w.Sq)
            T = int(cu[-1])
            q, k, v = make_qkv(1, w.H, T, T, w.D, seed=seed, Hkv=w.kv_heads)
            self.host = tuple(t[0].permute(1, 0, 2).contiguous() for t in (q, k, v))
            self.cu = cu.to(dev)
            self.maxlen = int(np.diff(cu.numpy()).max())
        else:
            self.host = make_qkv(w.B, w.H, w.Sq, w.Sk, w.D, seed=seed, Hkv=w.kv_heads)
        self.q, self.k, self.v = (t.to(dev).contiguous() for t in self.host)
        sl = alibi_slopes(w.H) if w.alibi else None
        doc = make_doc_ids(w.B, w.Sq) if w.doc else None
        self.sl = None if sl is None else sl.to(dev)
        self.doc = None if doc is None else doc.to(dev)
        if w.varlen:
            T = self.q.shape[0]
            self.o = torch.empty(T, w.H, w.D, dtype=torch.bfloat16, device=dev)
            self.lse = torch.empty(w.H, T, dtype=torch.float32, device=dev)
        else:
            self.o = torch.empty(w.B, w.H, w.Sq, w.D, dtype=torch.bfloat16, device=dev)
            self.lse = torch.empty(w.B, w.H, w.Sq, dtype=torch.float32, device=dev)
        self.launches_per_step = 2 if w.doc else 1
        if w.fp8:
            # e4m3 operands with per-128-row scales, quantised once (the quantiser is timed alone)
            self.q8 = [ta.attn_quantize_e4m3(t) for t in (self.q, self.k, self.v)]
        if w.fp4:
            # MXFP4 operands (V transposed), quantised once (the quantiser is timed alone)
            self.q4 = self.quantize_fp4(self.q, self.k, self.v)

    def quantize_fp4(self, q, k, v, out=None):
        ta = self.ta
        if out is None:
            return [ta.attn_quantize_mxfp4(q), ta.attn_quantize_mxfp4(k), ta.attn_quantize_mxfp4(v, transpose=True)]
        for t, tr, (xq, xs) in zip((q, k, v), (False, False, True), out):
            ta.attn_quantize_mxfp4(t, transpose=tr, xq=xq, x_sf=xs, stream=self.stream)
        return out

    def run(self, q, k, v, quantize=False):
        """The public call a user makes for this workload, on the given inputs."""
        w, ta = self.w, self.ta
        if w.fp4:
            a4 = self.quantize_fp4(q, k, v, out=self.q4) if quantize else self.q4
            (q4, qs), (k4, ks), (v4, vs) = a4
            ta.attn_fwd_fp4(q4, qs, k4, ks, v4, vs, w.Sk, o=self.o, lse=self.lse, scale=w.scale)
        elif w.fp8:
            if quantize:
                a8 = [ta.attn_quantize_e4m3(t) for t in (q, k, v)]
            else:
                a8 = self.q8
            (q8, qs), (k8, ks), (v8, vs) = a8
            ta.attn_fwd_fp8(q8, k8, v8, qs, ks, vs, o=self.o, lse=self.lse, scale=w.scale,
                            mask_kind=w.mask_kind)
        elif w.varlen:
            ta.attn_fwd_varlen(q, k, v, self.cu, self.cu, self.maxlen, self.maxlen, o=self.o, lse=self.lse,
                               scale=w.scale, mask_kind=w.mask_kind, window=w.window, softcap=w.softcap,
                               alibi_slopes=self.sl)
        else:
            ta.attn_fwd(q, k, v, o=self.o, lse=self.lse, scale=w.scale, mask_kind=w.mask_kind,
                        window=w.window, softcap=w.softcap, alibi_slopes=self.sl, doc_ids=self.doc)

    def step(self):
        self.run(self.q, self.k, self.v)

    def quantize_ms(self, reps=5):
        ta = self.ta
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(self.stream)
        for _ in range(reps):
            if self.w.fp4:
                self.quantize_fp4(self.q, self.k, self.v, out=self.q4)
                continue
            for t, (t8, ts) in zip((self.q, self.k, self.v), self.q8):
                ta.attn_quantize_e4m3(t, t8, ts, stream=self.stream)
        e1.record(self.stream)
        torch.cuda.synchronize(self.dev)
        return e0.elapsed_time(e1) / reps

    def tile_map_ms(self, reps=20):
        w, ta = self.w, self.ta
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(self.stream)
        for _ in range(reps):
            ta.attn_tile_map_build(w.B, w.Sq, w.Sk, w.mask_kind, w.window, doc_ids=self.doc, device=self.dev,
                                   stream=self.stream)
        e1.record(self.stream)
        torch.cuda.synchronize(self.dev)
        return e0.elapsed_time(e1) / reps


def time_launches(step, n, stream, dev, flush=None):
    """Per-launch device times (ms) of n eager steps, each bracketed by events on the
    launching stream; with ``flush`` (a buffer larger than L2) L2 is overwritten before every
    step.  Host work between the events counts, so this is for long steps only."""
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for i in range(n):
        if flush is not None:
            flush.add_(1)
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize(dev)
    return [s.elapsed_time(e) for s, e in zip(starts, ends)]


def capture(fn, n, dev):
    """A CUDA graph of n calls of fn (the calls run on torch's capture stream, which the
    library takes as the current stream), or None if capture is not possible."""
    try:
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            fn()
        torch.cuda.current_stream(dev).wait_stream(side)
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(n):
                fn()
        torch.cuda.synchronize(dev)
        return g
    except Exception as e:  # pragma: no cover - reported in the line as eager timing
        print(f"graph capture failed ({e}); timing eager launches", file=sys.stderr)
        torch.cuda.synchronize(dev)
        return None


def time_steps(step, n, dev, flush=None):
    """Device time (ms) of n steps replayed from one CUDA graph, bracketed by events: no host
    work between the launches.  With ``flush`` every step is preceded by an L2 flush inside
    the graph, and a graph of the flushes alone is timed and subtracted.  Returns
    (ms per step, "graph" | "eager")."""
    stream = torch.cuda.current_stream(dev)
    body = step if flush is None else (lambda: (flush.add_(1), step()))
    g = capture(body, n, dev)
    if g is None:
        ms = time_launches(step, n, stream, dev, flush)
        return float(np.mean(ms)), "eager"
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g.replay()                     # first replay uploads the graph
    torch.cuda.synchronize(dev)
    e0.record(stream)
    g.replay()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    total = e0.elapsed_time(e1)
    if flush is not None:
        gf = capture(lambda: flush.add_(1), n, dev)
        gf.replay()
        torch.cuda.synchronize(dev)
        e0.record(stream)
        gf.replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        total -= e0.elapsed_time(e1)
        del gf
    del g
    return total / n, "graph"


def compulsory_bytes(w) -> int:
    """Bytes each launch must move at least: Q, K, V read once, O and LSE written once."""
    if w.fp4:
        # e2m1 codes (V padded to 128 keys) and their 512-byte scale atoms per 128 rows or keys
        nq, nk = (w.Sq + 127) // 128, (w.Sk + 127) // 128
        qkv = w.B * (w.H * w.Sq * 64 + 2 * w.kv_heads * nk * 128 * 64)
        scales = w.B * (w.H * nq + 2 * w.kv_heads * nk) * 512
        return qkv + scales + w.B * w.H * w.Sq * (w.D * 2 + 4)
    eb = 1 if w.fp8 else 2
    qkv = w.B * (w.H * w.Sq + 2 * w.kv_heads * w.Sk) * w.D * eb
    scales = 3 * w.B * w.H * ((w.Sk + 127) // 128) * 4 if w.fp8 else 0
    return qkv + scales + w.B * w.H * w.Sq * (w.D * 2 + 4)


def per_config_record(ta, name, dev, peaks, min_ms=60.0, min_launches=10):
    """Device time, exact TFLOP/s, roofline fraction and (where profiled) DRAM traffic of one
    workload, measured alone after 3 warm-up launches."""
    w = WORKLOADS[name]
    case = Case(ta, w, dev, seed=0)
    for _ in range(3):
        case.step()
    torch.cuda.synchronize(dev)
    t1, _ = time_steps(case.step, 2, dev)
    n = max(min_launches, int(min_ms / max(t1, 1e-3)))
    flush = None
    if compulsory_bytes(w) < L2_BYTES:
        flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    mean_ms, how = time_steps(case.step, n, dev, flush)
    if ta.attn_get_status() != 0:
        raise SystemExit(f"kernel status error in workload {name}")
    flops = algorithmic_flops(w)
    tflops = flops / (mean_ms * 1e-3) / 1e12
    peak = peaks[peak_key(w)]
    gbs = compulsory_bytes(w) / (mean_ms * 1e-3) / 1e9
    rec = {"workload": w.note, "steps": n, "timing": how, "ms": mean_ms,
           "tflops_exact": tflops, "peak_tflops": peak, "frac": tflops / peak,
           "dtype": dtype_of(w), "compulsory_bytes": compulsory_bytes(w),
           "gbs_compulsory": gbs, "hbm_frac": gbs / peaks["hbm"],
           "l2": "flushed before every launch" if flush is not None else "inputs larger than L2",
           "traffic": profiled_traffic(name)}
    if w.doc:
        rec["tile_map_ms"] = case.tile_map_ms()
        rec["attention_ms"] = mean_ms - rec["tile_map_ms"]
    if w.fp4:
        rec["peak_source"] = peaks["fp4_source"]
    if w.fp8 or w.fp4:
        rec["quantize_ms_per_tensor_set"] = case.quantize_ms()
    del case, flush
    torch.cuda.empty_cache()
    return rec


def bwd_record(ta, name, dev, peaks, min_ms=60.0):
    """The backward of a workload (dQ, dK, dV from the forward's O and LSE and a random
    dO): device time of one attn_bwd call (its three launches) and TFLOP/s over the
    algorithmic 10 * D FLOPs per visible pair (five matrix products: Q K^T, dO V^T, P^T dO,
    dS^T Q, dS K; the kernels recompute two of them to avoid atomics, 14 * D done)."""
    w = WORKLOADS[name]
    case = Case(ta, w, dev, seed=0)
    case.step()
    g = torch.Generator().manual_seed(1)
    do = torch.randn(case.o.shape, generator=g).to(torch.bfloat16).to(dev)
    dq, dk, dv = (torch.empty_like(t) for t in (case.q, case.k, case.v))

    def bstep():
        ta.attn_bwd(case.q, case.k, case.v, case.o, case.lse, do, dq, dk, dv, scale=w.scale, mask_kind=w.mask_kind,
                    window=w.window, softcap=w.softcap, alibi_slopes=case.sl, doc_ids=case.doc)

    for _ in range(3):
        bstep()
    torch.cuda.synchronize(dev)
    t1, _ = time_steps(bstep, 2, dev)
    n = max(10, int(min_ms / max(t1, 1e-3)))
    mean_ms, how = time_steps(bstep, n, dev)
    if ta.attn_get_status() != 0:
        raise SystemExit(f"kernel status error in the backward of {name}")
    flops = 2.5 * algorithmic_flops(w)
    tflops = flops / (mean_ms * 1e-3) / 1e12
    rec = {"workload": w.note + ", backward", "steps": n, "timing": how, "ms": mean_ms, "tflops_exact": tflops,
           "peak_tflops": peaks["bf16"], "frac": tflops / peaks["bf16"],
           "flops": "10*D per visible pair (14*D executed: S and dP are recomputed for dQ)",
           "launches_per_call": 3}
    del case, do, dq, dk, dv
    torch.cuda.empty_cache()
    return rec


def sustained_record(case, dev, peaks, local, seconds=1.5):
    """Back-to-back launches for about ``seconds`` (long enough for the power cap to act),
    with its own NVML clock record, against the sustained peak."""
    t, _ = time_steps(case.step, 3, dev)
    per_graph = max(10, int(100.0 / max(t, 1e-3)))            # about 100 ms per replay
    reps = max(2, int(seconds * 1e3 / (per_graph * max(t, 1e-3))))
    g = capture(case.step, per_graph, dev)
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local, period_s=0.02) as clocks:
        e0.record(stream)
        for _ in range(reps):
            if g is not None:
                g.replay()
            else:
                for _ in range(per_graph):
                    case.step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1)
    n = reps * per_graph
    del g
    tflops = algorithmic_flops(case.w) * n / (ms * 1e-3) / 1e12
    peak = peaks[peak_key(case.w) + "_sustained"]
    return {"launches": n, "ms_total": ms, "tflops_exact": tflops, "peak_tflops": peak,
            "frac": tflops / peak if peak else None,
            "peak_source": "sustained GEMM peak (back-to-back loop under the power cap)",
            "clocks": clocks.summary()}


def measure_fp8_peak():
    """Dense e4m3 GEMM throughput on this GPU (torch._scaled_mm, 8192^3, bf16 output):
    burst = best of 10 single launches after warm-up, sustained = a 4 s back-to-back loop.
    Prints one JSON line; its numbers go to profiles/fp8_peak.json."""
    dev = torch.device("cuda", 0)
    n = 8192
    g = torch.Generator(device=dev).manual_seed(0)
    a = torch.randn(n, n, device=dev, generator=g).to(torch.float8_e4m3fn)
    b = torch.randn(n, n, device=dev, generator=g).to(torch.float8_e4m3fn).t()
    one = torch.ones((), device=dev)
    mm = lambda: torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
    for _ in range(10):
        mm()
    torch.cuda.synchronize()
    best = min(time_launches(mm, 10, torch.cuda.current_stream(), dev))
    flops = 2.0 * n ** 3
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = max(10, int(4000.0 / best))
    with ClockSampler(0, period_s=0.05) as clocks:
        e0.record()
        for _ in range(reps):
            mm()
        e1.record()
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    print(json.dumps({"fp8_tflops": flops / (best * 1e-3) / 1e12,
                      "fp8_tflops_sustained": flops * reps / (ms * 1e-3) / 1e12,
                      "method": "torch._scaled_mm e4m3 x e4m3 -> bf16, 8192^3; burst best of 10, "
                                f"sustained {reps} back to back ({ms / 1e3:.1f} s)",
                      "clocks": clocks.summary(), "gpu": torch.cuda.get_device_name(0)}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="causal", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true", help="skip the per-workload records")
    ap.add_argument("--measure-fp8-peak", action="store_true", help="time a dense e4m3 GEMM and exit")
    ap.add_argument("--kernel-only", action="store_true",
                    help="time the device steps only (no e2e, sustained, per-config or CPU legs): "
                         "the command the ncu captures run")
    ap.add_argument("--heads", type=int, default=0, help="override H (smaller ncu captures)")
    ap.add_argument("--backward", action="store_true",
                    help="with --kernel-only: time attn_bwd (dQ, dK, dV) of the workload instead of the forward")
    ap.add_argument("--pair", action="store_true",
                    help="with --kernel-only: time the forward through attn_fwd_pair (2-CTA clusters; "
                         "BF16 batched workloads with D = 128)")
    ap.add_argument("--tau", type=float, default=None,
                    help="ablation builds only (TILED_ATTENTION_LIB=.../libattn_abl*.so): rescale threshold; "
                         "the line then reports the rescale counters")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    w = WORKLOADS[args.workload]
    if args.heads > 0:
        import dataclasses
        w = dataclasses.replace(w, H=args.heads, note=w.note.replace(f"H{w.H}", f"H{args.heads}"))

    if args.pair and (not args.kernel_only or args.backward or w.fp8 or w.fp4 or w.varlen or w.D != 128):
        ap.error("--pair needs --kernel-only and a BF16 batched forward workload with D = 128")
    if args.backward and (not args.kernel_only or w.fp8 or w.fp4 or w.varlen):
        ap.error("--backward needs --kernel-only and a BF16 batched workload")

    if args.impl == "reference":
        run_reference(args, w)
        return
    if args.measure_fp8_peak:
        measure_fp8_peak()
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    import tiled_attention_14_b200 as ta
    lib = ta._lib.load()
    dev = torch.device("cuda", local)
    ablation = None
    if args.tau is not None:
        import ctypes
        lib.attn_ablation_set.restype, lib.attn_ablation_set.argtypes = ctypes.c_int, [ctypes.c_float]
        lib.attn_ablation_counts.restype, lib.attn_ablation_counts.argtypes = ctypes.c_int, [ctypes.c_void_p]
        lib.attn_ablation_sw_exp_every.restype = ctypes.c_int
        ablation = {"tau": args.tau, "sw_exp_every": lib.attn_ablation_sw_exp_every(),
                    "lib": os.path.basename(os.environ.get("TILED_ATTENTION_LIB", ""))}
    case = Case(ta, w, dev, seed=rank)
    stream = torch.cuda.current_stream(dev)
    quant_ms = case.quantize_ms() if (w.fp8 or w.fp4) else None
    if args.pair:
        def pair_step():
            ta.attn_fwd_pair(case.q, case.k, case.v, o=case.o, lse=case.lse, scale=w.scale, mask_kind=w.mask_kind,
                             window=w.window, softcap=w.softcap, alibi_slopes=case.sl, doc_ids=case.doc)
        case.step = pair_step
    if args.backward:
        case.step()
        g = torch.Generator().manual_seed(1)
        do = torch.randn(case.o.shape, generator=g).to(torch.bfloat16).to(dev)
        grads = [torch.empty_like(t) for t in (case.q, case.k, case.v)]

        def bwd_step():
            ta.attn_bwd(case.q, case.k, case.v, case.o, case.lse, do, *grads, scale=w.scale,
                        mask_kind=w.mask_kind, window=w.window, softcap=w.softcap, alibi_slopes=case.sl,
                        doc_ids=case.doc)
        case.step = bwd_step
        case.launches_per_step = 3 + (1 if w.doc else 0)

    for _ in range(args.warmup):
        case.step()
    torch.cuda.synchronize(dev)
    if ta.attn_get_status(stream) != 0:
        raise SystemExit("kernel status error during warm-up")
    if ablation is not None:
        if lib.attn_ablation_set(args.tau) != 0:
            raise SystemExit("attn_ablation_set failed")

    # The K timed steps are one CUDA graph (captured after the warm-up, not timed), so the
    # device runs them back to back with no host work between launches.
    graph = capture(case.step, args.steps, dev)
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t_begin = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        t_begin.record(stream)
        if graph is not None:
            graph.replay()
        else:
            for _ in range(args.steps):
                case.step()
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    if dist:
        dist.barrier()
    total_ms = t_begin.elapsed_time(t_end)
    timing = "cuda graph of the K steps" if graph is not None else "eager launches"
    del graph
    if ta.attn_get_status(stream) != 0:
        raise SystemExit("kernel status error in the timed region")

    flops = algorithmic_flops(w) * (2.5 if args.backward else 1.0)
    total_ms = max_over_ranks(total_ms, dist, dev)
    value = weak_scaling_value(flops, args.steps, world, total_ms)
    if ablation is not None:
        import ctypes
        cnt = (ctypes.c_ulonglong * 2)()
        if lib.attn_ablation_counts(ctypes.addressof(cnt)) != 0:
            raise SystemExit("attn_ablation_counts failed")
        ablation.update(rescale_steps_per_launch=cnt[0] / args.steps, row_steps_per_launch=cnt[1] / args.steps,
                        rescale_fraction=cnt[0] / max(cnt[1], 1))
    if args.kernel_only:
        if rank == 0:
            line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
                    "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
                    "config": workload_config(w), "kernel_only": True, "backward": args.backward,
                    "pair": args.pair,
                    "gpu_launches": case.launches_per_step * args.steps}
            if ablation is not None:
                line["ablation"] = ablation
            print(json.dumps(line), flush=True)
        if dist:
            dist.barrier()
            dist.destroy_process_group()
        return

    # ---- end to end through the public API: pinned host inputs in, host outputs back
    qh, kh, vh = (t.pin_memory() for t in case.host)
    oh = torch.empty(case.o.shape, dtype=case.o.dtype).pin_memory()
    lh = torch.empty(case.lse.shape, dtype=case.lse.dtype).pin_memory()
    q2, k2, v2 = (torch.empty_like(t) for t in (case.q, case.k, case.v))

    def e2e_step():
        q2.copy_(qh, non_blocking=True)
        k2.copy_(kh, non_blocking=True)
        v2.copy_(vh, non_blocking=True)
        case.run(q2, k2, v2, quantize=True)
        oh.copy_(case.o, non_blocking=True)
        lh.copy_(case.lse, non_blocking=True)

    e2e_steps = max(3, min(args.steps, 20))
    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize(dev)
    if dist:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    e2e_value = weak_scaling_value(flops, e2e_steps, world, e2e_ms)
    h2d = sum(t.numel() * t.element_size() for t in case.host)
    d2h = case.o.numel() * case.o.element_size() + case.lse.numel() * case.lse.element_size()
    del q2, k2, v2, qh, kh, vh, oh, lh

    if rank == 0:
        peaks = measured_peaks()
        # the attention kernel is the dominant launch (one launch per step for analytic masks)
        launch_ms = total_ms / args.steps
        achieved = flops / (launch_ms * 1e-3) / 1e12
        peak = peaks[peak_key(w)]
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": dtype_of(w),
            "data": "synthetic", "config": {**workload_config(w), "parallelism": f"replicas x{world}"},
            "tflops_tile_count": weak_scaling_value(tile_count_flops(w), args.steps, world, total_ms),
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": profiled_traffic(args.workload),
                         "peak_source": (peaks["fp4_source"] if w.fp4 else peaks["fp8_source"] if w.fp8 else
                                         f"bf16_tflops of {peaks['source']} peaks (burst)")
                                        + f"; bf16 sustained {peaks['bf16_sustained']}",
                         "kernel": "attn_fp4_kernel" if w.fp4 else "attn_fwd_kernel",
                         "algorithmic_flops_per_launch": flops},
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "clocks": clocks.summary(),
            "gpu_launches": case.launches_per_step * args.steps,
            "timing": timing,
        }
        if quant_ms is not None:
            line["quantize_ms_per_tensor_set"] = quant_ms
        if world == 1 and not args.no_per_config:
            # each workload alone, before the seconds-long sustained loop heats the part
            line["per_config"] = {}
            for name in WORKLOADS:
                time.sleep(0.5)
                with ClockSampler(local, period_s=0.01) as cs:
                    rec = per_config_record(ta, name, dev, peaks)
                rec["clocks"] = cs.summary()
                line["per_config"][name] = rec
            with ClockSampler(local, period_s=0.01) as cs:
                rec = bwd_record(ta, "causal", dev, peaks)
            rec["clocks"] = cs.summary()
            line["per_config"]["causal_backward"] = rec
        if world == 1:
            line["sustained"] = sustained_record(case, dev, peaks, local)
        if world == 1 and not args.no_cpu_baseline:
            f, dt, desc = oracle_sample(w, args.cpu_budget)
            line["cpu_baseline"] = {"value": f / dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(),
                                    "kind": "oracle", "sample": desc}
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
