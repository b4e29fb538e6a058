"""FP4 (e2m1) code book, MX block quantiser and the Direct-P attention forward — oracle
(test infrastructure only).

Follows "Hardware-Aware FP4 FlashAttention-4" (gist.science): the summary paragraph (a
forward pass for non-causal inference that runs on Blackwell's FP4 tensor cores, up to
2.13x faster) and the Direct-P paragraphs (rather than computing each probability and
then scaling and rounding it to FP4, the raw scores are mapped straight onto the codes the
hardware multiplies).  The page names neither the element format, nor the block scaling,
nor the mapping itself.  The readings taken here:

Element format: e2m1 — 1 sign bit, 2 exponent bits with bias 1, 1 mantissa bit; exponent
field 0 holds the subnormal 0.5; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 for codes 0..7,
code + 8 the negatives; no infinity or NaN.  Encoding: round to nearest, ties to the even
code, saturating at +-6 (the PTX ``cvt.rn.satfinite.e2m1x2.f32`` behaviour).

Block scaling of Q, K and V (OCP Microscaling, MXFP4): one power-of-two scale 2^X per 32
consecutive elements along the contraction axis (D for Q and K, the keys for V), stored
as the E8M0 byte X + 127.  X = floor(log2 amax) - 2, 2 being the largest e2m1 exponent,
clamped to [-127, 127]; an all-zero block stores X = -127.  Element = encode(x / 2^X).

Direct-P (the encoder of P): the score of row i and key j in log2 units is
t_ij = scale * log2(e) * (q_i . k_j), with q, k the dequantised inputs.  Keys form blocks
of 32 (j // 32), the block scale of P.  For each row and block, E = floor(max t over the
block's keys) - 2, and each key gets the code

    c = clip(rint(2 (t - E) + 2), 0, 7)        (rint: nearest integer, ties to even)

i.e. the e2m1 codes read as a logarithmic scale in half octaves (code 2 is 2^0, code 4 is
2^1, code 6 is 2^2, the odd codes between them): the code is the score itself, rounded to
the nearest half octave, with no exponential and no rounding of a probability in between.
P~_ij = value(c) * 2^E, the e2m1 magnitude the tensor core multiplies (the odd codes' 1.5
sits 0.085 octave above the half-octave point they stand for), represents 2^t_ij.
Attention then normalises by what it multiplied:

    O_i = sum_j P~_ij v_j / sum_j P~_ij,    LSE_i = ln(sum_j P~_ij).

Keys at or beyond Sk are not part of any block maximum and contribute nothing.
"""
from __future__ import annotations

import math

import numpy as np

BLOCK = 32                       # elements per MX scale (Q, K along D; V and P along keys)
E2M1_MAX = 6.0
LOG2E = 1.0 / math.log(2.0)


def code_values() -> np.ndarray:
    """float64 value of each of the 16 e2m1 codes, from the bit fields."""
    vals = np.empty(16, dtype=np.float64)
    for code in range(16):
        sign = -1.0 if code & 0x8 else 1.0
        e = (code >> 1) & 0x3
        m = code & 0x1
        vals[code] = sign * (0.5 * m if e == 0 else (1.0 + 0.5 * m) * 2.0 ** (e - 1))
    return vals


VALUES = code_values()
_POS = VALUES[:8]                # 0, 0.5, 1, 1.5, 2, 3, 4, 6: code order is value order


def encode(x) -> np.ndarray:
    """Round-to-nearest-even, saturating e2m1 encoding of a float array -> uint8 codes 0..15.

    The input is taken exactly (as float64).  The sign bit is the input's, as in IEEE
    conversions: -0 and negative values that round to zero give code 8 (-0)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E2M1_MAX)
    lo = np.clip(np.searchsorted(_POS, a, side="right") - 1, 0, 7)
    hi = np.minimum(lo + 1, 7)
    dlo = a - _POS[lo]
    dhi = _POS[hi] - a
    up = (dhi < dlo) | ((dhi == dlo) & (lo % 2 == 1) & (hi != lo))
    c = np.where(up, hi, lo).astype(np.uint8)
    neg = np.signbit(x)
    return np.where(neg, c | 0x8, c).astype(np.uint8)


def decode(codes) -> np.ndarray:
    return VALUES[np.asarray(codes, dtype=np.int64)]


def mx_quantize(x, axis: int = -1):
    """MXFP4 quantisation along ``axis`` in blocks of 32 (the axis length is zero-padded to a
    multiple of 32).  Returns (codes uint8 same shape as the padded x, X int32 with the axis
    divided by 32).  x is taken as float32 values (exactly, as float64)."""
    x = np.moveaxis(np.asarray(x, dtype=np.float32).astype(np.float64), axis, -1)
    n = x.shape[-1]
    npad = -n % BLOCK
    if npad:
        x = np.concatenate([x, np.zeros(x.shape[:-1] + (npad,))], axis=-1)
    blocks = x.reshape(x.shape[:-1] + (-1, BLOCK))
    amax = np.abs(blocks).max(axis=-1)
    _, e = np.frexp(np.where(amax > 0, amax, 1.0))      # amax = f * 2^e, f in [0.5, 1)
    X = np.where(amax > 0, e - 1 - 2, -127)
    X = np.clip(X, -127, 127).astype(np.int32)
    codes = encode(blocks / np.ldexp(1.0, X)[..., None])
    codes = codes.reshape(x.shape)
    return np.moveaxis(codes, -1, axis), np.moveaxis(X, -1, axis)


def mx_dequantize(codes, X, axis: int = -1) -> np.ndarray:
    """Inverse of ``mx_quantize``: value(code) * 2^X, float64, padded length."""
    c = np.moveaxis(np.asarray(codes), axis, -1)
    Xm = np.moveaxis(np.asarray(X), axis, -1)
    vals = decode(c).reshape(c.shape[:-1] + (-1, BLOCK))
    out = vals * np.ldexp(1.0, Xm.astype(np.int64))[..., None]
    return np.moveaxis(out.reshape(c.shape), -1, axis)


def direct_p_codes(t, E) -> np.ndarray:
    """Direct-P code of scores t (log2 units) against block exponents E (broadcast)."""
    y2 = 2.0 * (np.asarray(t, dtype=np.float64) - np.asarray(E, dtype=np.float64)) + 2.0
    return np.clip(np.rint(y2), 0, 7).astype(np.int64)


def direct_p_rows(t: np.ndarray):
    """Direct-P weights of score rows t [R, Sk] (log2 units; -inf marks keys that take no
    part).  Returns (P~ [R, Sk], codes [R, Sk], E [R, nblocks])."""
    R, Sk = t.shape
    npad = -Sk % BLOCK
    tp = np.concatenate([t, np.full((R, npad), -np.inf)], axis=1) if npad else t
    blocks = tp.reshape(R, -1, BLOCK)
    bmax = blocks.max(axis=2)
    live = np.isfinite(bmax)
    E = np.where(live, np.floor(np.where(live, bmax, 0.0)) - 2.0, 0.0)
    codes = direct_p_codes(np.where(np.isfinite(blocks), blocks, -1e300), E[:, :, None])
    codes = np.where(np.isfinite(blocks), codes, 0)
    ptil = _POS[codes] * np.ldexp(1.0, E.astype(np.int64))[:, :, None]
    ptil = ptil.reshape(R, -1)[:, :Sk]
    return ptil, codes.reshape(R, -1)[:, :Sk], E


def attention_fp4_fwd(q, k, v, scale: float, rows=None):
    """Direct-P attention, no mask, on dequantised inputs q [B,H,Sq,D], k/v [B,Hkv,Sk,D]
    (float64, H a multiple of Hkv).  Returns (O [B,H,R,D], LSE [B,H,R]) for the query rows
    ``rows`` (all rows if None)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, H, Sq, D = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    G = H // Hkv
    rows = np.arange(Sq) if rows is None else np.asarray(rows, dtype=np.int64)
    O = np.zeros((B, H, len(rows), D))
    L = np.zeros((B, H, len(rows)))
    for b in range(B):
        for h in range(H):
            t = (q[b, h, rows] @ k[b, h // G].T) * (float(scale) * LOG2E)
            ptil, _, _ = direct_p_rows(t)
            l = ptil.sum(axis=1)
            O[b, h] = (ptil @ v[b, h // G]) / l[:, None]
            L[b, h] = np.log(l)
    return O, L
