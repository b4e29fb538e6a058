"""Error floor of the FP8 path's P rounding — a diagnostic of the test suite, not the oracle.

The FP8 forward of config 5 rounds the softmax weights P to e4m3 before P.V (page
"FlashAttention-3: Rekordverdächtige Geschwindigkeit und Präzision bei AI-Modellen",
section "Analyse": FP8 with block quantisation).  That rounding is part of the method, so
the output differs from the exact softmax of the dequantised inputs by an amount the
kernel cannot remove.  This module computes, from the oracle's own pieces:

* ``rounded_p_output``: the output when P is rounded to e4m3 the way the FP8 path reads it
  (P = exp(s - m) with the V block's scale folded in as sV[kt] / max(sV), then e4m3; the
  row sum uses the unrounded P).  ``c`` multiplies P before the rounding and divides it out
  after, as a running maximum that trails the true maximum by log2(c) does in the kernel.
* ``rounding_bounds``: per output element, a worst-case bound W and a standard deviation
  sigma of that rounding error.  Each weight x_j = c p_j sV/max(sV) is moved by at most
  h_j = max(2^-4 x_j, 2^-10) (half a unit in the last place of e4m3: 3 mantissa bits in
  the normal range, spacing 2^-9 among the subnormals), so
      W     = max(sV) / (c l) * sum_j h_j |vcode_j|
      sigma = max(sV) / (c l) * sqrt(sum_j h_j^2 vcode_j^2 / 3)
  (errors uniform in [-h_j, h_j]).  Both shrink as c grows, so the bounds at c = 1 hold for
  every running maximum the kernel may use.

The GPU tests bound the kernel's error per element by 5e-2 + min(W, 6 sigma) + 2^-8 |O|.
"""
from __future__ import annotations

import numpy as np

from oracle import e4m3
from oracle.attention import modified_scores, visible_mask

E4M3_HALF_ULP_REL = 2.0 ** -4
E4M3_HALF_SUBNORMAL_STEP = 2.0 ** -10


def _weights(q, k, scale, rows, Sq, Sk, mask_kind, window):
    """Unnormalised softmax weights p = exp(s - m) (0 where masked) and row sums, fp64."""
    vis = visible_mask(rows, Sq, Sk, mask_kind, window, None)
    s = modified_scores(q[rows], k, scale, rows, Sq, Sk, 0.0, None)
    s = np.where(vis, s, -np.inf)
    m = s.max(axis=1)
    m = np.where(np.isfinite(m), m, 0.0)
    p = np.where(vis, np.exp(s - m[:, None]), 0.0)
    return p, p.sum(axis=1)


def head_inputs(qc, qs, kc, ks, vc, vs):
    """Dequantised q, k and the V codes' values with the per-key V block scale, for one
    (b, h): codes [S, D] uint8 and scales [nblocks]."""
    rep = lambda s, n: np.repeat(np.asarray(s, np.float64), e4m3.BLOCK_ROWS)[:n]
    q = e4m3.decode(qc) * rep(qs, qc.shape[0])[:, None]
    k = e4m3.decode(kc) * rep(ks, kc.shape[0])[:, None]
    vcode = e4m3.decode(vc)
    sv = rep(vs, vc.shape[0])
    return q, k, vcode, sv


def rounded_p_output(q, k, vcode, sv, scale, rows, mask_kind=0, window=0, c=1.0):
    """Output rows with P rounded to e4m3 (V block scale folded in), fp64 [R, D]."""
    Sq, Sk = q.shape[0], k.shape[0]
    p, l = _weights(q, k, scale, rows, Sq, Sk, mask_kind, window)
    vnorm = float(sv.max())
    x = c * p * (sv / vnorm)[None, :]
    xq = e4m3.decode(e4m3.encode(x))
    out = (xq @ vcode) * (vnorm / c)
    return np.divide(out, l[:, None], out=np.zeros_like(out), where=l[:, None] > 0)


def rounding_bounds(q, k, vcode, sv, scale, rows, mask_kind=0, window=0):
    """(W, sigma, E_p|v|) per output element [R, D] for the rounding of P at c = 1."""
    Sq, Sk = q.shape[0], k.shape[0]
    p, l = _weights(q, k, scale, rows, Sq, Sk, mask_kind, window)
    vnorm = float(sv.max())
    x = p * (sv / vnorm)[None, :]
    h = np.where(p > 0, np.maximum(E4M3_HALF_ULP_REL * x, E4M3_HALF_SUBNORMAL_STEP), 0.0)
    inv = np.divide(vnorm, l, out=np.zeros_like(l), where=l > 0)[:, None]
    W = (h @ np.abs(vcode)) * inv
    sigma = np.sqrt((h * h) @ (vcode * vcode) / 3.0) * inv
    w = np.divide(p, l[:, None], out=np.zeros_like(p), where=l[:, None] > 0)
    e_abs_v = w @ np.abs(vcode * sv[:, None])
    return W, sigma, e_abs_v
