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
                            doc_lengths, make_doc_ids, make_fp8_source, make_qkv)

METRIC = "attention fwd TFLOP/s and % of B200 dense BF16/FP8 tensor peak, per config"
L2_BYTES = 126 * 1024 * 1024


# ----------------------------------------------------------------------------- FLOP counts
def visible_pairs(w) -> int:
    """Exact number of visible (i, j) pairs over the whole batch (all b, h)."""
    Sq, Sk = w.Sq, w.Sk
    d = Sk - Sq
    if w.mask_kind & MASK_DOC:
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
    if w.mask_kind & MASK_DOC:
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
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"bf16": d["bf16_tflops"], "bf16_sustained": d.get("bf16_tflops_sustained"),
                "hbm": d["hbm_gbs"], "source": "measured"}
    return {"bf16": 1590.0, "bf16_sustained": 1400.0, "hbm": 6650.0, "source": "fallback"}


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


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "tiled_attention_14_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per launch of the attention kernel from the committed ncu summary, if the
    kernel source has not changed since it was captured."""
    p = os.path.join(ROOT, "profiles", f"traffic_{workload}.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    if d.get("kernel_source_hash") != kernel_source_hash():
        return None
    return d.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------- CPU oracle leg
def oracle_sample(w, budget_s: float, seed: int = 0):
    """Times the fp64 oracle on the workload until about budget_s of CPU work is done:
    whole (b, h) heads while one head fits the budget, else an evenly spaced subset of one
    head's query rows.  Returns (algorithmic FLOPs done, seconds, description)."""
    from oracle.attention import attention_fwd, visible_mask
    q, k, v = make_qkv(1, 1, w.Sq, w.Sk, w.D, seed=seed)
    sl = alibi_slopes(w.H)[:1].numpy() if w.alibi else None
    doc = make_doc_ids(1, w.Sq) if w.doc else None
    doc_np = None if doc is None else doc[0].numpy()

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
    return {"workload": w.note, "B": w.B, "H": w.H, "Sq": w.Sq, "Sk": w.Sk, "D": w.D,
            "mask": {"causal": bool(w.mask_kind & MASK_CAUSAL), "window": w.window,
                     "alibi": w.alibi, "softcap": w.softcap, "document": w.doc},
            "flops": "exact: 4*D per visible (i,j) pair",
            "l2": f"inputs larger than L2 ({(3 * w.B * w.H * w.Sk * w.D * 2) / 1e6:.0f} MB of Q/K/V + "
                  f"{w.B * w.H * w.Sq * w.D * 2 / 1e6:.0f} MB of O vs 126 MB L2); no flush"}


# ----------------------------------------------------------------------------- GPU leg
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="causal", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    w = WORKLOADS[args.workload]

    if args.impl == "reference":
        run_reference(args, w)
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
    ta._lib.load()

    if w.fp8:
        q, k, v = make_fp8_source(w.B, w.H, w.Sq, w.D, seed=rank)
    else:
        q, k, v = make_qkv(w.B, w.H, w.Sq, w.Sk, w.D, seed=rank)
    sl = alibi_slopes(w.H) if w.alibi else None
    doc = make_doc_ids(w.B, w.Sq) if w.doc else None
    dev = torch.device("cuda", local)
    qd, kd, vd = (t.to(dev).contiguous() for t in (q, k, v))
    sld = None if sl is None else sl.to(dev)
    docd = None if doc is None else doc.to(dev)
    o = torch.empty(w.B, w.H, w.Sq, w.D, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(w.B, w.H, w.Sq, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    launches_per_step = 2 if w.doc else 1

    quant_ms = None
    if w.fp8:
        # e4m3 operands with per-128-row scales, quantised once; the quantiser is timed alone
        q8, qs = ta.attn_quantize_e4m3(qd, stream=stream)
        k8, ks = ta.attn_quantize_e4m3(kd, stream=stream)
        v8, vs = ta.attn_quantize_e4m3(vd, stream=stream)
        e0q, e1q = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0q.record(stream)
        for t, (t8, ts) in zip((qd, kd, vd), ((q8, qs), (k8, ks), (v8, vs))):
            ta.attn_quantize_e4m3(t, t8, ts, stream=stream)
        e1q.record(stream)
        torch.cuda.synchronize(dev)
        quant_ms = e0q.elapsed_time(e1q)

    def step():
        if w.fp8:
            ta.attn_fwd_fp8(q8, k8, v8, qs, ks, vs, o=o, lse=lse, scale=w.scale, mask_kind=w.mask_kind,
                            stream=stream)
        else:
            ta.attn_fwd(qd, kd, vd, o=o, lse=lse, scale=w.scale, mask_kind=w.mask_kind, window=w.window,
                        softcap=w.softcap, alibi_slopes=sld, doc_ids=docd, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if ta.attn_get_status(stream) != 0:
        raise SystemExit("kernel status error during warm-up")

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t_begin = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        t_begin.record(stream)
        for i in range(args.steps):
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    if dist:
        dist.barrier()
    total_ms = t_begin.elapsed_time(t_end)
    per_launch_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    if ta.attn_get_status(stream) != 0:
        raise SystemExit("kernel status error in the timed region")

    flops = algorithmic_flops(w)
    total_ms = max_over_ranks(total_ms, dist, dev)
    value = weak_scaling_value(flops, args.steps, world, total_ms)

    # ---- end to end through the public API: pinned host inputs in, host outputs back
    qh, kh, vh = (t.pin_memory() for t in (q, k, v))
    oh = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    lh = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    q2, k2, v2 = (torch.empty_like(t) for t in (qd, kd, vd))

    def e2e_step():
        q2.copy_(qh, non_blocking=True)
        k2.copy_(kh, non_blocking=True)
        v2.copy_(vh, non_blocking=True)
        if w.fp8:
            a8 = [ta.attn_quantize_e4m3(t, stream=stream) for t in (q2, k2, v2)]
            ta.attn_fwd_fp8(a8[0][0], a8[1][0], a8[2][0], a8[0][1], a8[1][1], a8[2][1], o=o, lse=lse,
                            scale=w.scale, mask_kind=w.mask_kind, stream=stream)
        else:
            ta.attn_fwd(q2, k2, v2, o=o, lse=lse, scale=w.scale, mask_kind=w.mask_kind, window=w.window,
                        softcap=w.softcap, alibi_slopes=sld, doc_ids=docd, stream=stream)
        oh.copy_(o, non_blocking=True)
        lh.copy_(lse, non_blocking=True)

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
    h2d = sum(t.numel() * t.element_size() for t in (q, k, v))
    d2h = o.numel() * o.element_size() + lse.numel() * lse.element_size()

    if rank == 0:
        peaks = measured_peaks()
        # the attention kernel is the dominant launch; its time per launch is the event
        # time per step minus nothing else for analytic masks (one launch per step)
        launch_ms = float(np.mean(per_launch_ms))
        achieved = flops / (launch_ms * 1e-3) / 1e12
        # FP8 contractions take the FP8 peak: the measured BF16 peak times the nominal
        # dense FP8 / BF16 ratio (4.5 / 2.25 PFLOP/s)
        peak = peaks["bf16"] * (2.0 if w.fp8 else 1.0)
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "e4m3" if w.fp8 else "bf16",
            "data": "synthetic", "config": {**workload_config(w), "parallelism": f"replicas x{world}"},
            "tflops_tile_count": weak_scaling_value(tile_count_flops(w), args.steps, world, total_ms),
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "traffic": profiled_traffic(args.workload),
                         "peak_source": (f"bf16_tflops of {peaks['source']} peaks (burst)"
                                         + (" x 2 (nominal fp8/bf16)" if w.fp8 else "")
                                         + f"; bf16 sustained {peaks['bf16_sustained']}"),
                         "kernel": "attn_fwd_kernel", "algorithmic_flops_per_launch": flops},
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "clocks": clocks.summary(),
            "gpu_launches": launches_per_step * args.steps,
        }
        if quant_ms is not None:
            line["quantize_ms_per_tensor_set"] = quant_ms
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
