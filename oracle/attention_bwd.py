"""Plain fp64 attention backward — the oracle (test infrastructure only).

What it computes
----------------
The gradients dQ, dK, dV of a scalar loss L through the attention forward of
``oracle.attention.attention_fwd``, given dO = dL/dO.  The pages compare FA4's backward
passes with cuDNN's and note that block-sparse backward runs are not deterministic
(page "PyTorch's FlexAttention mit FlashAttention-4 ist ein Game-Changer", sections
"Leistung und Validierung" and "Aktuelle Einschränkungen"; the same section says captured
tensors such as learnable biases get no gradient, so the ALiBi slopes get none here); the
page "FlashAttention 4: ..." lists the backward pass among FA4's missing parts (section
"Κύρια Συμπεράσματα").  The pages give no formula, so this is the chain rule applied to the
forward definition, step by step in the forward's order reversed:

    s   = scale * q_i . k_j                       (scores)
    t   = c * tanh(s / c)   if soft-capping        (score_mod, first)
    t  += slope_h * (j - i')  if ALiBi             (score_mod, second; no gradient to slope)
    P   = softmax over the visible j of t          (masked entries: P = 0)
    O   = P V

    dV  = P^T dO
    dP  = dO V^T
    dT  = P * (dP - Dv),  Dv_i = sum_j P_ij dP_ij  (= sum_d dO_id O_id)
    dS  = dT * (1 - tanh^2(s / c))  if soft-capping, else dT
    dQ  = scale * dS K,   dK = scale * dS^T Q

Grouped-query attention (Hkv < H): key/value head g serves query heads g*G .. g*G+G-1
(G = H / Hkv), so its dK and dV are the sums over those query heads.  A query row with no
visible key has P = 0 and contributes nothing.  Rows are taken in chunks; nothing is
tiled or reordered beyond that.
"""
from __future__ import annotations

import numpy as np

from .attention import MASK_DOC, _f64, modified_scores, softmax_rows, visible_mask


def attention_bwd(q, k, v, do, scale: float, mask_kind: int = 0, window: int = 0,
                  softcap: float = 0.0, alibi_slopes=None, doc_ids=None, chunk: int = 512):
    """fp64 gradients (dQ [B,H,Sq,D], dK [B,Hkv,Sk,D], dV [B,Hkv,Sk,D]).

    q, do: [B,H,Sq,D]; k, v: [B,Hkv,Sk,D]; other arguments as attention_fwd."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, H, Sq, D = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    if H % Hkv != 0:
        raise ValueError("the number of key/value heads must divide the number of query heads")
    G = H // Hkv
    if mask_kind & MASK_DOC and Sq != Sk:
        raise ValueError("document mask needs Sq == Sk")
    slopes = None if alibi_slopes is None else _f64(alibi_slopes).reshape(-1)
    docs = None if doc_ids is None else np.asarray(
        doc_ids.cpu().numpy() if hasattr(doc_ids, "cpu") else doc_ids)
    dQ = np.zeros_like(q)
    dK = np.zeros_like(k)
    dV = np.zeros_like(v)
    rows_all = np.arange(Sq, dtype=np.int64)
    for b in range(B):
        doc_row = None if docs is None else docs[b]
        for r0 in range(0, Sq, chunk):
            rr = rows_all[r0:r0 + chunk]
            vis = visible_mask(rr, Sq, Sk, mask_kind, window, doc_row)
            for h in range(H):
                hk = h // G
                slope = None if slopes is None else slopes[h]
                t = modified_scores(q[b, h, rr], k[b, hk], scale, rr, Sq, Sk, softcap, slope)
                P, _, _ = softmax_rows(t, vis)
                dO = do[b, h, rr]
                dV[b, hk] += P.T @ dO
                dP = dO @ v[b, hk].T
                Dv = (P * dP).sum(axis=1, keepdims=True)
                dT = P * (dP - Dv)
                if softcap and softcap > 0:
                    s = (q[b, h, rr] @ k[b, hk].T) * float(scale)
                    th = np.tanh(s / float(softcap))
                    dS = dT * (1.0 - th * th)
                else:
                    dS = dT
                dQ[b, h, rr] = float(scale) * (dS @ k[b, hk])
                dK[b, hk] += float(scale) * (dS.T @ q[b, h, rr])
    return dQ, dK, dV
