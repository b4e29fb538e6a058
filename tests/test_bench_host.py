"""Host logic of bench.py (CPU only): exact FLOP counts against the oracle's brute-force
visible-pair count, and the reference (oracle) arm's JSON line."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

import bench
from attn_workloads import MASK_CAUSAL, MASK_DOC, MASK_NONE, MASK_WINDOW, Workload, doc_ids_from_lengths, doc_lengths
from oracle.attention import visible_pair_count

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("Sq,Sk,mask,W", [(300, 300, MASK_NONE, 0), (300, 300, MASK_CAUSAL, 0),
                                          (200, 520, MASK_CAUSAL, 0), (520, 200, MASK_CAUSAL, 0),
                                          (700, 700, MASK_CAUSAL | MASK_WINDOW, 128),
                                          (700, 650, MASK_WINDOW, 77)])
def test_visible_pairs_match_oracle(Sq, Sk, mask, W):
    w = Workload("t", 2, 3, Sq, Sk, 64, mask, window=W)
    assert bench.visible_pairs(w) == 6 * visible_pair_count(Sq, Sk, mask, W)


@pytest.mark.parametrize("mask", [MASK_DOC, MASK_DOC | MASK_CAUSAL])
def test_visible_pairs_documents(mask):
    w = Workload("d", 2, 2, 8192, 8192, 128, mask, doc=True)
    ref = sum(visible_pair_count(8192, 8192, mask, 0, doc_ids_from_lengths(doc_lengths(8192, b)))
              for b in range(2)) * 2
    assert bench.visible_pairs(w) == ref


def test_benchmark_flop_counts():
    assert bench.algorithmic_flops(bench.WORKLOADS["causal"]) == 4 * 128 * 64 * (4096 * 4097 // 2)
    assert bench.algorithmic_flops(bench.WORKLOADS["long"]) == 4 * 128 * 32 * 32768 ** 2
    # the kernel's 256x128 tiles cover a little more than the exact causal half
    w = bench.WORKLOADS["causal"]
    assert bench.tile_count_flops(w) > bench.algorithmic_flops(w)


def test_reference_arm_prints_one_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny", "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, timeout=300, check=True).stdout
    lines = [l for l in out.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0


@pytest.mark.parametrize("argv", [["--pair"], ["--pair", "--kernel-only", "--workload", "fp8"],
                                  ["--pair", "--kernel-only", "--workload", "tiny"],
                                  ["--pair", "--kernel-only", "--backward"], ["--backward"],
                                  ["--backward", "--kernel-only", "--workload", "varlen"]])
def test_mode_flags_rejected_before_any_device_use(argv):
    """--pair and --backward need --kernel-only and a workload the entry point takes; the
    error comes from the argument check (exit 2), before any GPU work."""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + argv, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 2, (r.returncode, r.stderr[-300:])
    assert "needs --kernel-only" in r.stderr


def test_committed_traffic_files_are_well_formed():
    """Every profiles/traffic_<workload>.json names a known workload, a kernel source hash
    and positive DRAM byte counts whose sum is the per-launch figure."""
    pdir = os.path.join(ROOT, "profiles")
    files = [f for f in os.listdir(pdir) if f.startswith("traffic_") and f.endswith(".json")]
    assert files
    for f in files:
        d = json.load(open(os.path.join(pdir, f)))
        assert f == f"traffic_{d['workload']}.json" and d["workload"] in bench.WORKLOADS
        assert len(d["kernel_source_hash"]) == 16
        # a small output can stay in L2 for the whole capture (no DRAM write)
        assert d["dram_bytes_read"] > 0 and d["dram_bytes_write"] >= 0
        assert d["dram_bytes_per_launch"] == d["dram_bytes_read"] + d["dram_bytes_write"]


def test_profiled_traffic_is_gated_by_the_kernel_source_hash(tmp_path, monkeypatch):
    """A traffic figure is reported only while the kernel sources' code (comments aside) matches
    the capture."""
    csrc = tmp_path / "tiled_attention_14_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in bench.FWD_SOURCES:
        (csrc / f).write_text("// source\n")
    (csrc / "attn_fwd_kernel.cuh").write_text("// kernel\nint v = 1;\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.kernel_source_hash()
    rec = {"workload": "causal", "kernel_source_hash": h, "dram_bytes_per_launch": 123.0}
    (tmp_path / "profiles" / "traffic_causal.json").write_text(json.dumps(rec))
    assert bench.profiled_traffic("causal") == 123.0
    assert bench.profiled_traffic("long") is None              # no capture for this workload
    (csrc / "attn_bwd_kernel.cuh").write_text("// another kernel\n")   # not part of the forward
    assert bench.profiled_traffic("causal") == 123.0
    (csrc / "attn_fwd_kernel.cuh").write_text("/* kernel */ // edited comment\n\nint v = 1;  // here\n")
    assert bench.profiled_traffic("causal") == 123.0          # comments and blank lines only
    (csrc / "attn_fwd_kernel.cuh").write_text("// kernel\nint v = 2;\n")   # the kernel changed since
    assert bench.profiled_traffic("causal") is None


def test_profiled_traffic_hash_is_per_kernel_family(tmp_path, monkeypatch):
    """An FP4 kernel change invalidates the FP4 capture only; a change to the sources both
    families share invalidates both."""
    csrc = tmp_path / "tiled_attention_14_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in bench.FP4_SOURCES:
        (csrc / f).write_text(f"int {f.split('.')[0]} = 1;\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    for wl, fam in (("causal", "bf16"), ("fp4_long", "fp4")):
        rec = {"workload": wl, "kernel_source_hash": bench.kernel_source_hash(fam), "dram_bytes_per_launch": 7.0}
        (tmp_path / "profiles" / f"traffic_{wl}.json").write_text(json.dumps(rec))
    assert bench.kernel_source_hash("bf16") != bench.kernel_source_hash("fp4")
    assert bench.profiled_traffic("causal") == 7.0 and bench.profiled_traffic("fp4_long") == 7.0
    (csrc / "attn_fp4_kernel.cuh").write_text("int attn_fp4_kernel = 2;\n")
    assert bench.profiled_traffic("causal") == 7.0 and bench.profiled_traffic("fp4_long") is None
    (csrc / "ptx.cuh").write_text("int ptx = 2;\n")
    assert bench.profiled_traffic("causal") is None


def test_fp4_workload_accounting():
    """FP4 long: the algorithmic FLOPs of the BF16 long shape, compulsory bytes of the e2m1 codes
    (V padded to 128 keys), the scale atoms, O and LSE, and the FP4 peak as FP8 x 2."""
    w = bench.WORKLOADS["fp4_long"]
    assert w.fp4 and not w.fp8 and w.mask_kind == 0
    assert bench.algorithmic_flops(w) == bench.algorithmic_flops(bench.WORKLOADS["long"])
    nq = nk = 32768 // 128
    expect = 32 * 32768 * 64 + 2 * 32 * nk * 128 * 64 + 32 * (nq + 2 * nk) * 512 + 32 * 32768 * (128 * 2 + 4)
    assert bench.compulsory_bytes(w) == expect
    assert bench.dtype_of(w) == "e2m1" and bench.peak_key(w) == "fp4"
    peaks = bench.measured_peaks()
    assert peaks["fp4"] == 2 * peaks["fp8"]
