"""Build libattn.so in-tree with nvcc for sm_100a.

    python -m tiled_attention_14_b200.build      (or call build())

The shared library is written next to this file, so that it travels with the source tree.
"""
from __future__ import annotations

import os
import re
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libattn.so")
SOURCES = ["attn_api.cu"]


def _nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _deps() -> list[str]:
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files += [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE)]
    return files


# Ablation builds (test and measurement only, never the product path): the same sources with
# ATTN_ABLATION (runtime rescale threshold, rescale counters, include/attn_ablation.h) and
# optionally the software exp2 on one element pair in four.
ABLATIONS = {
    "libattn_abl.so": ["-DATTN_ABLATION"],
    "libattn_abl_sw4.so": ["-DATTN_ABLATION", "-DATTN_SW_EXP_EVERY=4"],
}


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in _deps())


# Debug build (tests only): every TMA copy and TMEM move bounds-checked in the kernels, a failed
# check recorded as ATTN_ERR_CHECK in the status word instead of a fault.
DEBUG = {"libattn_debug.so": ["-DATTN_DEBUG_CHECKS"]}


def build_ablations(force: bool = False, verbose: bool = False) -> list[str]:
    """Builds the ablation libraries and the bounds-checked debug library."""
    out = []
    for name, flags in {**ABLATIONS, **DEBUG}.items():
        out.append(build(force=force, verbose=verbose, extra=flags, lib=os.path.join(HERE, name)))
    return out


def build(force: bool = False, verbose: bool = False, extra: list[str] | None = None, lib: str = LIB) -> str:
    if not force and up_to_date(lib):
        return lib
    LIB_OUT = lib
    tmp = LIB_OUT + ".tmp"
    cmd = [_nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
           "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
           "-I", INCLUDE, "-I", CSRC, "--expt-relaxed-constexpr",
           "-o", tmp] + [os.path.join(CSRC, s) for s in SOURCES] + list(extra or [])
    cmd += ["-Xptxas", "-v"]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed")
    check_registers(res.stderr)
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(tmp, LIB_OUT)
    return LIB_OUT


# Registers per thread the attention kernels must be compiled to: the kernel's setmaxnreg
# split (softmax warpgroups up, producer/MMA warpgroup down) adds up to exactly this many
# per thread at launch, so any other count is a build error.
LAUNCH_REGS = 168


def check_registers(ptxas_log: str) -> None:
    entry = None
    seen = 0
    for line in ptxas_log.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            entry = m.group(1)
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and entry and "attn_fwd_kernel" in entry:
            n = int(m.group(1))
            if n != LAUNCH_REGS:
                raise RuntimeError(f"{entry}: ptxas assigned {n} registers, the register split needs {LAUNCH_REGS}")
            seen += 1
            entry = None
    if seen == 0:
        raise RuntimeError("no attention kernel found in the ptxas report")


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="--ptxas-v" in sys.argv)
    if "--ablations" in sys.argv:
        build_ablations(force="--force" in sys.argv)
