"""Test infrastructure for the FP4 forward (not part of the oracle): the storage layout the
C-ABI uses for MXFP4 tensors, written from the layout the header states, and the
per-element bound of the Direct-P kernel against the fp64 oracle.

Why a bound and not equality: the kernel decides each P code from its fp32 score (the
tensor core's fp32 accumulation of exact FP4 products); the oracle decides it from the fp64
score.  Where a score sits within the fp32 accumulation error of a code boundary — or a
block maximum within it of an integer (the block exponent) — the two may pick neighbouring
codes, and both are correct readings of the definition.  The bound adds, for every such
ambiguous element, the largest change of P~ the other choice makes, carried through
O = sum P~ v / sum P~ to first order (|dO_d| <= sum |dP~_j| |v_jd - O_d| / L), plus the bf16
rounding of O.  A wrong code rule, scale or layout moves O far outside it.
"""
from __future__ import annotations

import math

import numpy as np

from oracle import fp4

# fp32 accumulation of the 128 exact products: |error| <= 128 * 2^-24 * sum |q_d k_d|; the
# window is taken 16x wider than that.
SCORE_REL_ERR = 2.0 ** -13


def pack_rows(codes: np.ndarray) -> np.ndarray:
    """[..., n] codes (0..15) -> [..., n/2] bytes, element 2i in the low nibble of byte i."""
    c = codes.astype(np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def sf_atoms(X: np.ndarray, nrows_valid: int) -> np.ndarray:
    """Block exponents X [..., R, 4] (R rows of a 128-row-padded operand, 4 blocks per row)
    -> E8M0 atoms [..., R/128, 512]: row r of an atom, block k at byte 16 (r % 32) +
    4 (r // 32) + k; rows at or past nrows_valid get byte 0."""
    lead = X.shape[:-2]
    R = X.shape[-2]
    assert R % 128 == 0 and X.shape[-1] == 4
    out = np.zeros(lead + (R // 128, 512), dtype=np.uint8)
    for r in range(R):
        a, rr = divmod(r, 128)
        off = 16 * (rr % 32) + 4 * (rr // 32)
        if r < nrows_valid:
            out[..., a, off:off + 4] = (X[..., r, :] + 127).astype(np.uint8)
    return out


def expected_rows(x: np.ndarray):
    """Oracle MXFP4 of Q or K as the C-ABI stores it: (codes [B,H,S,64], atoms [B,H,nt,512])."""
    B, H, S, D = x.shape
    codes, X = fp4.mx_quantize(x.astype(np.float32), axis=-1)
    nt = (S + 127) // 128
    Xp = np.zeros((B, H, nt * 128, 4), dtype=np.int64)
    Xp[:, :, :S] = X
    return pack_rows(codes), sf_atoms(Xp, S)


def expected_transposed(v: np.ndarray):
    """Oracle MXFP4 of V stored transposed: (codes [B,H,128,Sp/2], atoms [B,H,Sp/128,512])."""
    B, H, S, D = v.shape
    Sp = (S + 127) // 128 * 128
    vp = np.zeros((B, H, Sp, D), dtype=np.float32)
    vp[:, :, :S] = v
    vt = np.swapaxes(vp, -1, -2)                    # [B, H, 128, Sp]
    codes, X = fp4.mx_quantize(vt, axis=-1)         # X [B, H, 128, Sp/32]
    nt = Sp // 128
    atoms = np.zeros((B, H, nt, 512), dtype=np.uint8)
    for kt in range(nt):
        Xk = X[:, :, :, 4 * kt:4 * kt + 4]         # [B, H, 128 (d), 4]
        atoms[:, :, kt] = sf_atoms(Xk, 128)[:, :, 0]
    return pack_rows(codes), atoms


def dequantised(q, k, v):
    """fp64 Q^, K^, V^ [B, H, S, 128] from the oracle quantiser."""
    out = []
    for x in (q, k):
        c, X = fp4.mx_quantize(np.asarray(x, dtype=np.float32), axis=-1)
        out.append(fp4.mx_dequantize(c, X, axis=-1)[..., :x.shape[-1]])
    # V is quantised along the keys (its contraction axis), not along D
    vt = np.swapaxes(np.asarray(v, dtype=np.float32), -1, -2)
    c, X = fp4.mx_quantize(vt, axis=-1)
    vh = np.swapaxes(fp4.mx_dequantize(c, X, axis=-1)[..., :vt.shape[-1]], -1, -2)
    return out[0], out[1], vh


def _alt_ptilde(t, E, lo, hi):
    """P~ of scores t under block exponent E with the code clipped to [lo, hi]."""
    c = np.clip(np.rint(2.0 * (t - E) + 2.0), lo, hi)
    c = np.clip(c, 0, 7).astype(np.int64)
    return fp4.VALUES[c] * np.ldexp(1.0, E.astype(np.int64))


def reference_with_bound(qh, kh, vh, scale, rows):
    """(O, LSE, bound_O, bound_LSE) for the query rows `rows` of every (b, h); qh [B,H,Sq,D],
    kh/vh [B,Hkv,Sk,D] dequantised fp64."""
    B, H, Sq, D = qh.shape
    Hkv, Sk = kh.shape[1], kh.shape[2]
    G = H // Hkv
    c = float(scale) / math.log(2.0)
    R = len(rows)
    O = np.zeros((B, H, R, D))
    L = np.zeros((B, H, R))
    bO = np.zeros((B, H, R, D))
    bL = np.zeros((B, H, R))
    for b in range(B):
        for h in range(H):
            q = qh[b, h, rows]
            kk = kh[b, h // G]
            vv = vh[b, h // G]
            t = (q @ kk.T) * c
            dt = SCORE_REL_ERR * (np.abs(q) @ np.abs(kk).T) * c + 1e-30
            ptil, codes, E = fp4.direct_p_rows(t)
            l = ptil.sum(axis=1)
            o = (ptil @ vv) / l[:, None]
            # elements near a code boundary: 2(t - E) + 2 within 2 dt of a half integer
            nb = E.shape[1]
            Ef = np.repeat(E, fp4.BLOCK, axis=1)[:, :Sk]
            y2 = 2.0 * (t - Ef) + 2.0
            near = np.abs(y2 - np.floor(y2) - 0.5) < 2.0 * dt
            up = np.abs(_alt_ptilde(t + dt, Ef, 0, 7) - ptil)
            down = np.abs(_alt_ptilde(t - dt, Ef, 0, 7) - ptil)
            dp = np.where(near, np.maximum(up, down), 0.0)
            # blocks whose maximum is near an integer: the whole block may use E - 1 or E + 1
            pad = -Sk % fp4.BLOCK
            tp = np.concatenate([t, np.full((R, pad), -np.inf)], axis=1) if pad else t
            dtp = np.concatenate([dt, np.zeros((R, pad))], axis=1) if pad else dt
            bmax = tp.reshape(R, nb, fp4.BLOCK).max(axis=2)
            bdt = dtp.reshape(R, nb, fp4.BLOCK).max(axis=2)
            frac = bmax - np.floor(bmax)
            amb = np.isfinite(bmax) & ((frac < bdt) | (1.0 - frac < bdt))
            if amb.any():
                for Eshift in (-1.0, 1.0):
                    Ealt = np.repeat(E + Eshift, fp4.BLOCK, axis=1)[:, :Sk]
                    alt = _alt_ptilde(t, Ealt, 0, 7)
                    m = np.repeat(amb, fp4.BLOCK, axis=1)[:, :Sk]
                    dp = np.where(m, np.maximum(dp, np.abs(alt - ptil) + np.maximum(up, down)), dp)
            dl = dp.sum(axis=1)
            bO[b, h] = (dp @ np.abs(vv)) / l[:, None] + np.abs(o) * (dl / l)[:, None]
            bL[b, h] = dl / l
            O[b, h] = o
            L[b, h] = np.log(l)
    return O, L, bO, bL
