"""FP8 e4m3 code book, encoder and per-block quantiser — oracle (test infrastructure only).

The FP8 path follows the page "FlashAttention-3: Rekordverdächtige Geschwindigkeit und
Präzision bei AI-Modellen", section "Analyse" (FP8 with block quantisation, to keep
accuracy in the presence of outlier features).  The pages give neither the block size
nor the format; the benchmark configuration fixes e4m3 with one fp32 scale per 128
consecutive rows of each (b, h).

Format (OCP FP8 E4M3, "fn" variant): 1 sign bit, 4 exponent bits with bias 7, 3
mantissa bits; exponent field 0 holds subnormals m/8 * 2^-6; code 0x7F / 0xFF is NaN;
there is no infinity, the largest finite magnitude is 448 (exponent field 15, mantissa 6).

Encoding reading: round to nearest, ties to the even code, saturate finite values beyond
the largest magnitude to +-448 (the PTX ``cvt.rn.satfinite.e4m3x2.f32`` behaviour).

Block quantiser reading: for each (b, h, block of 128 rows): a = max |x| over the block
(fp32); stored scale = a / 448 and multiplier = 448 / a, each one correctly rounded fp32
division; code = encode(fp32(x * multiplier)).  A block of zeros stores scale 1 and
multiplier 1.  The dequantised value is decode(code) * scale.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
BLOCK_ROWS = 128


def code_values() -> np.ndarray:
    """float64 value of each of the 256 codes (NaN for 0x7F and 0xFF)."""
    vals = np.empty(256, dtype=np.float64)
    for code in range(256):
        sign = -1.0 if code & 0x80 else 1.0
        e = (code >> 3) & 0xF
        m = code & 0x7
        if e == 0xF and m == 0x7:
            vals[code] = np.nan
        elif e == 0:
            vals[code] = sign * (m / 8.0) * 2.0 ** (-6)
        else:
            vals[code] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


_VALS = code_values()
# Non-negative finite codes 0x00..0x7E in increasing value order (code order is value order).
_POS_CODES = np.arange(0x7F, dtype=np.int64)
_POS_VALS = _VALS[:0x7F]


def encode(x) -> np.ndarray:
    """Round-to-nearest-even, saturating e4m3 encoding of a float array -> uint8 codes.

    The input is taken exactly (as float64).  NaN maps to 0x7F."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    sat = a >= E4M3_MAX
    a_c = np.minimum(a, E4M3_MAX)
    # index of the largest grid value <= a
    lo = np.searchsorted(_POS_VALS, a_c, side="right") - 1
    lo = np.clip(lo, 0, len(_POS_VALS) - 1)
    hi = np.minimum(lo + 1, len(_POS_VALS) - 1)
    vlo = _POS_VALS[lo]
    vhi = _POS_VALS[hi]
    dlo = a_c - vlo
    dhi = vhi - a_c
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi != lo) & (_POS_CODES[lo] % 2 == 1))
    mag = np.where(pick_hi, _POS_CODES[hi], _POS_CODES[lo])
    mag = np.where(sat, 0x7E, mag)
    code = np.where(np.signbit(x), mag | 0x80, mag)
    code = np.where(np.isnan(x), 0x7F, code)
    return code.astype(np.uint8)


def decode(codes) -> np.ndarray:
    """uint8 codes -> float64 values."""
    return _VALS[np.asarray(codes, dtype=np.int64)]


def quantize_blocks(x) -> tuple[np.ndarray, np.ndarray]:
    """fp32 [B,H,S,D] -> (codes uint8 [B,H,S,D], scales fp32 [B,H,ceil(S/128)])."""
    x = np.asarray(x.detach().cpu().numpy() if hasattr(x, "detach") else x, dtype=np.float32)
    B, H, S, D = x.shape
    nb = (S + BLOCK_ROWS - 1) // BLOCK_ROWS
    codes = np.empty(x.shape, dtype=np.uint8)
    scales = np.empty((B, H, nb), dtype=np.float32)
    for blk in range(nb):
        r0, r1 = blk * BLOCK_ROWS, min(S, (blk + 1) * BLOCK_ROWS)
        xb = x[:, :, r0:r1, :]
        amax = np.abs(xb).max(axis=(2, 3)).astype(np.float32)          # [B,H]
        zero = amax == 0
        safe = np.where(zero, np.float32(1.0), amax).astype(np.float32)
        scale = np.where(zero, np.float32(1.0), safe / np.float32(E4M3_MAX)).astype(np.float32)
        mult = np.where(zero, np.float32(1.0), np.float32(E4M3_MAX) / safe).astype(np.float32)
        y = (xb * mult[:, :, None, None]).astype(np.float32)           # fp32 product, rn
        codes[:, :, r0:r1, :] = encode(y)
        scales[:, :, blk] = scale
    return codes, scales


def dequantize_blocks(codes, scales) -> np.ndarray:
    """(codes [B,H,S,D], scales [B,H,nb]) -> float64 [B,H,S,D] = decode(code) * scale."""
    codes = np.asarray(codes)
    scales = np.asarray(scales, dtype=np.float64)
    S = codes.shape[2]
    rep = np.repeat(scales, BLOCK_ROWS, axis=2)[:, :, :S]
    return decode(codes) * rep[..., None]
