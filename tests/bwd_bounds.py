"""Per-element error bounds of the bf16 backward kernels against the fp64 oracle (test
infrastructure, not part of the oracle).

The kernels take Q, K, V, dO in bf16 and O, LSE from the bf16 forward, accumulate in fp32,
and round three things to bf16: P (the dV operand), P * dt/ds and dS (the dK and dQ
operands), and the outputs.  With P, dP, Dv and dS from the oracle's definitions, each
gradient element g is held to

    |g_kernel - g| <= eps * T + 2^-8 |g| + atol

where T is the sum of the absolute values of the terms that make g up (rounding of each
term cannot move g by more than its relative error times T) plus the effect of the
forward output's own rounding on Dv (O is bf16: |dDv_i| <= 2^-8 sum_d |dO_id O_id|):

    dV_j :  T = sum_i P_ij |dO_i|
    dK_j :  T = scale * sum_i (|dS_ij| + P_ij f'_ij A_i) |Q_i|,   A_i = sum_d |dO_id O_id|
    dQ_i :  T = scale * sum_j (|dS_ij| + P_ij f'_ij A_i) |K_j|

eps = 2^-7 + 2^-10 covers two bf16 roundings of a term (half an ulp, 2^-8 each: bf16 keeps
8 significant bits) and the LSE error of the forward (about 1e-6 in natural-log units).  A wrong or dropped term moves g by about |g|
itself, far outside the bound.
"""
from __future__ import annotations

import numpy as np

from oracle.attention import _f64, modified_scores, softmax_rows, visible_mask
from oracle.attention_bwd import attention_bwd

EPS = 2.0 ** -7 + 2.0 ** -10
REL_OUT = 2.0 ** -8
ATOL = 1e-5


def bwd_bounds(q, k, v, do, scale, mask_kind=0, window=0, softcap=0.0, alibi_slopes=None, doc_ids=None):
    """(dQ, dK, dV) from the oracle and their per-element bounds (same shapes)."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    dq, dk, dv = attention_bwd(q, k, v, do, scale, mask_kind, window, softcap, alibi_slopes, doc_ids)
    B, H, Sq, D = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    G = H // Hkv
    slopes = None if alibi_slopes is None else _f64(alibi_slopes).reshape(-1)
    docs = None if doc_ids is None else np.asarray(doc_ids.cpu().numpy() if hasattr(doc_ids, "cpu") else doc_ids)
    Tq = np.zeros_like(dq)
    Tk = np.zeros_like(dk)
    Tv = np.zeros_like(dv)
    rows = np.arange(Sq)
    for b in range(B):
        vis = visible_mask(rows, Sq, Sk, mask_kind, window, None if docs is None else docs[b])
        for h in range(H):
            hk = h // G
            t = modified_scores(q[b, h], k[b, hk], scale, rows, Sq, Sk, softcap,
                                None if slopes is None else slopes[h])
            P, _, _ = softmax_rows(t, vis)
            O = P @ v[b, hk]
            dP = do[b, h] @ v[b, hk].T
            Dv = (P * dP).sum(axis=1, keepdims=True)
            if softcap and softcap > 0:
                th = np.tanh((q[b, h] @ k[b, hk].T) * scale / softcap)
                fp = 1.0 - th * th
            else:
                fp = np.ones_like(P)
            dS = P * (dP - Dv) * fp
            A = (np.abs(do[b, h]) * np.abs(O)).sum(axis=1, keepdims=True)
            W = np.abs(dS) + P * fp * A
            Tv[b, hk] += P.T @ np.abs(do[b, h])
            Tk[b, hk] += scale * (W.T @ np.abs(q[b, h]))
            Tq[b, h] = scale * (W @ np.abs(k[b, hk]))
    bound = lambda T, g: EPS * T + REL_OUT * np.abs(g) + ATOL
    return (dq, dk, dv), (bound(Tq, dq), bound(Tk, dk), bound(Tv, dv))
