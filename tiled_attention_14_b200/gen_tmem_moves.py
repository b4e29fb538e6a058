"""Writes csrc/tmem_moves.cuh: the TMEM <-> register moves of the attention kernels.

    python -m tiled_attention_14_b200.gen_tmem_moves          (rewrites the header)
    python -m tiled_attention_14_b200.gen_tmem_moves --check  (exit 1 if it is stale)

Each move is one `tcgen05.ld` / `tcgen05.st` of the 32x32b shape with n 32-bit registers,
so its inline-PTX operand list is long and regular; it is written out by this script rather
than by hand.  Loads carry their `tcgen05.wait::ld` in the same asm statement; stores come
in a `_nowait` and a `_wait` form and take a compile-time slice of a register array.
"""
from __future__ import annotations

import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
OUT = os.path.join(HERE, "csrc", "tmem_moves.cuh")

LOAD_WIDTHS = (16, 32, 64, 128)
STORE_WIDTHS = (16, 32, 64)

HEADER = """#pragma once
#include <cstdint>

namespace attn {

// TMEM <-> register moves (32x32b shape: thread t of the warp moves lane 32*(warp%4)+t).
// Loads wrap the asynchronous move and its wait in ONE asm statement so that no use of
// the registers can be scheduled between them.  Stores take a compile-time slice
// r[OFF .. OFF+n) of a register array; the _nowait form must be followed by a _wait
// store (or tcgen05.wait::st) before the data is handed to the tensor core, and the
// stored registers are not rewritten before that.
"""

FOOTER = """
}  // namespace attn
"""


# In the debug build (ATTN_DEBUG_CHECKS) each move first checks its TMEM column range and lane
# quarter (tmem_range_ok, ptx.cuh); a failed check is recorded and the move skipped (a load
# then returns zeros).
def _check(n: int, load: bool) -> str:
    fill = f"    for (int i = 0; i < {n}; ++i) r[i] = 0u;\n" if load else ""
    return (
        "#ifdef ATTN_DEBUG_CHECKS\n"
        f"  if (!debug_check(tmem_range_ok(taddr, {n}))) {{\n"
        f"{fill}"
        "    return;\n"
        "  }\n"
        "#endif\n")


def _load(n: int) -> str:
    regs = ", ".join(f"%{i}" for i in range(n))
    outs = ", ".join(f'"=r"(r[{i}])' for i in range(n))
    return (
        f"__device__ __forceinline__ void tmem_ld_x{n}_wait(uint32_t taddr, uint32_t (&r)[{n}]) {{\n"
        + _check(n, True) +
        f"  asm volatile(\n"
        f'    "tcgen05.ld.sync.aligned.32x32b.x{n}.b32 {{{regs}}}, [%{n}];\\n\\t"\n'
        f'    "tcgen05.wait::ld.sync.aligned;\\n"\n'
        f"    : {outs}\n"
        f'    : "r"(taddr) : "memory");\n'
        f"}}\n")


def _store(n: int, wait: bool) -> str:
    regs = ", ".join(f"%{i + 1}" for i in range(n))
    ins = ", ".join(f'"r"(r[OFF + {i}])' for i in range(n))
    name = f"tmem_st_x{n}_{'wait' if wait else 'nowait'}"
    wait_line = '    "tcgen05.wait::st.sync.aligned;\\n"\n' if wait else ""
    return (
        f"template <int OFF, int N>\n"
        f"__device__ __forceinline__ void {name}(uint32_t taddr, const uint32_t (&r)[N]) {{\n"
        f'  static_assert(OFF + {n} <= N, "slice out of range");\n'
        + _check(n, False) +
        f"  asm volatile(\n"
        f'    "tcgen05.st.sync.aligned.32x32b.x{n}.b32 [%0], {{{regs}}};\\n\\t"\n'
        f"{wait_line}"
        f'    :: "r"(taddr), {ins}\n'
        f'    : "memory");\n'
        f"}}\n")


def render() -> str:
    parts = [HEADER]
    parts += [_load(n) for n in LOAD_WIDTHS]
    for n in STORE_WIDTHS:
        parts.append(_store(n, wait=False))
        parts.append(_store(n, wait=True))
    parts.append(FOOTER)
    return "".join(parts)


def main(argv: list[str]) -> int:
    text = render()
    if "--check" in argv:
        current = open(OUT).read() if os.path.exists(OUT) else ""
        return 0 if current == text else 1
    with open(OUT, "w") as f:
        f.write(text)
    return 0


if __name__ == "__main__":
    sys.exit(main(sys.argv[1:]))
