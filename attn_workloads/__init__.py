"""Seeded synthetic inputs for the attention forward pass.

This module is shared by the fp64 oracle's tests, the CUDA parity tests and the
benchmark.  It only draws random numbers and lays out the workload shapes; it holds
none of the attention arithmetic (no scores, no softmax, no quantisation), so the two
implementations that it feeds stay independent.

The workloads are the ones the FlexAttention / FlashAttention pages speak of:
plain SDPA (page "FlashAttention 4", section "Εισαγωγή"), the FlexAttention variants
causal, sliding window, ALiBi, soft-capping and document masking (page "PyTorch's
FlexAttention mit FlashAttention-4", intro), and FP8 inputs with outlier features
(page "FlashAttention-3", analysis paragraph on FP8 and block quantisation).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

# Mask bit flags of the C-ABI (include/attn.h).  Kept here as plain data so that the
# harness can name them; the oracle defines its own copy.
MASK_NONE = 0
MASK_CAUSAL = 1
MASK_WINDOW = 2
MASK_DOC = 4


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    Sq: int
    Sk: int
    D: int
    mask_kind: int = MASK_NONE
    window: int = 0
    softcap: float = 0.0
    alibi: bool = False
    doc: bool = False
    fp8: bool = False
    fp4: bool = False        # MXFP4 Q/K/V from the bf16 inputs, Direct-P forward (non-causal)
    note: str = ""
    Hkv: int = 0             # key/value heads (0: same as H)
    varlen: bool = False     # packed sequences with the document lengths of doc_lengths()

    @property
    def kv_heads(self) -> int:
        return self.Hkv or self.H

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)


# The five benchmark configurations (the fourth one is split into its four variants,
# the fifth into its non-causal and causal runs).
WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 256, 256, 64, note="B1 H2 S256 D64 non-causal"),
    "causal": Workload("causal", 4, 16, 4096, 4096, 128, MASK_CAUSAL,
                       note="B4 H16 S4096 D128 causal"),
    "window": Workload("window", 2, 16, 8192, 8192, 128, MASK_CAUSAL | MASK_WINDOW, window=1024,
                       note="B2 H16 S8192 D128 sliding window 1024, causal"),
    "alibi": Workload("alibi", 2, 16, 8192, 8192, 128, MASK_CAUSAL, alibi=True,
                      note="B2 H16 S8192 D128 ALiBi + causal"),
    "softcap": Workload("softcap", 2, 16, 8192, 8192, 128, MASK_NONE, softcap=50.0,
                        note="B2 H16 S8192 D128 tanh softcap 50, non-causal"),
    "doc": Workload("doc", 2, 16, 8192, 8192, 128, MASK_DOC, doc=True,
                    note="B2 H16 S8192 D128 document mask, lengths U[256,2048]"),
    "long": Workload("long", 1, 32, 32768, 32768, 128, note="B1 H32 S32768 D128 non-causal"),
    "fp4_long": Workload("fp4_long", 1, 32, 32768, 32768, 128, fp4=True,
                         note="B1 H32 S32768 D128 non-causal, MXFP4 Q/K/V, Direct-P"),
    "fp8": Workload("fp8", 2, 16, 16384, 16384, 128, fp8=True,
                    note="B2 H16 S16384 D128 FP8 e4m3, non-causal"),
    "fp8_causal": Workload("fp8_causal", 2, 16, 16384, 16384, 128, MASK_CAUSAL, fp8=True,
                           note="B2 H16 S16384 D128 FP8 e4m3, causal"),
    # Beyond the five configurations: grouped-query heads and packed sequences (the two
    # gaps the FA4 page names), on shapes of the configurations above.
    "gqa": Workload("gqa", 4, 32, 4096, 4096, 128, MASK_CAUSAL, Hkv=8,
                    note="B4 H32 Hkv8 S4096 D128 causal (grouped-query heads)"),
    "varlen": Workload("varlen", 2, 16, 8192, 8192, 128, MASK_NONE, varlen=True,
                       note="2 x 8192 tokens packed as sequences of lengths U[256,2048], H16 D128"),
}


def varlen_cu_seqlens(B: int, S: int) -> torch.Tensor:
    """int32 [nseq + 1] offsets of the sequences of ``doc_lengths(S, seed=b)`` for b < B,
    packed one batch row after another."""
    lens = [n for b in range(B) for n in doc_lengths(S, b)]
    return torch.from_numpy(np.concatenate([[0], np.cumsum(lens)]).astype(np.int32))


def make_qkv(B: int, H: int, Sq: int, Sk: int, D: int, seed: int = 0,
             dtype: torch.dtype = torch.bfloat16, q_mul: float = 1.0, Hkv: int = 0):
    """Q, K, V drawn i.i.d. N(0,1) on the CPU from one torch generator, in the order
    q, k, v, then cast to ``dtype``.  Layout [B, H, S, D] ([B, Hkv, Sk, D] for K and V
    when Hkv is given), contiguous."""
    g = torch.Generator().manual_seed(seed)
    hk = Hkv or H
    q = torch.randn(B, H, Sq, D, generator=g)
    k = torch.randn(B, hk, Sk, D, generator=g)
    v = torch.randn(B, hk, Sk, D, generator=g)
    if q_mul != 1.0:
        q = q * q_mul
    return q.to(dtype), k.to(dtype), v.to(dtype)


def doc_lengths(S: int, seed: int, lo: int = 256, hi: int = 2048) -> list[int]:
    """Document lengths for one batch row: uniform integers in [lo, hi] that sum to S.

    While more than ``hi`` tokens remain, draw U{lo .. min(hi, rem - lo)} (so the
    remainder never falls below ``lo``); the last document takes the rest."""
    rng = np.random.default_rng(seed)
    out, rem = [], S
    while rem > 0:
        if rem <= hi:
            out.append(rem)
            break
        n = int(rng.integers(lo, min(hi, rem - lo) + 1))
        out.append(n)
        rem -= n
    return out


def doc_ids_from_lengths(lengths: list[int]) -> np.ndarray:
    """Running document index per token (int32)."""
    return np.repeat(np.arange(len(lengths), dtype=np.int32), lengths)


def make_doc_ids(B: int, S: int, lo: int = 256, hi: int = 2048) -> torch.Tensor:
    """int32 [B, S]: batch row b uses ``doc_lengths(S, seed=b)``."""
    rows = [doc_ids_from_lengths(doc_lengths(S, b, lo, hi)) for b in range(B)]
    return torch.from_numpy(np.stack(rows)).to(torch.int32)


def alibi_slopes(H: int) -> torch.Tensor:
    """ALiBi slopes 2^(-8(h+1)/H), h = 0..H-1, as fp32 [H]."""
    return torch.tensor([2.0 ** (-8.0 * (h + 1) / H) for h in range(H)], dtype=torch.float32)


def make_fp8_source(B: int, H: int, S: int, D: int, seed: int = 0, frac: float = 0.001,
                    factor: float = 20.0):
    """fp32 Q, K, V ~ N(0,1) with outlier channels.

    For each tensor independently, ``max(1, round(frac*H*D))`` of the H*D hidden
    channels (h, d), chosen by ``torch.randperm`` on the same generator, are multiplied
    by ``factor`` for every b and s."""
    g = torch.Generator().manual_seed(seed)
    out = []
    for _ in range(3):
        x = torch.randn(B, H, S, D, generator=g)
        n_out = max(1, int(round(frac * H * D)))
        idx = torch.randperm(H * D, generator=g)[:n_out]
        for c in idx.tolist():
            h, d = divmod(c, D)
            x[:, h, :, d] *= factor
        out.append(x)
    return tuple(out)


def sample_rows(Sq: int, n_random: int, seed: int, extra: list[int] | None = None) -> np.ndarray:
    """Query rows for sampled checks at full size: the first two rows, the last row,
    tile edges (multiples of 128 and their predecessors), any ``extra`` rows, and
    ``n_random`` seeded random rows.  Sorted, unique, all < Sq."""
    rows = {0, 1, Sq - 1}
    for t in range(128, Sq, 128 * max(1, (Sq // 128) // 8)):
        rows.update((t - 1, t))
    if extra:
        rows.update(r for r in extra if 0 <= r < Sq)
    rng = np.random.default_rng(seed)
    rows.update(int(r) for r in rng.integers(0, Sq, size=n_random))
    return np.array(sorted(r for r in rows if 0 <= r < Sq), dtype=np.int64)
