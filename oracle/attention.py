"""Plain fp64 attention forward — the oracle (test infrastructure only).

Definition followed
-------------------
* Scaled dot-product attention: queries are multiplied with keys, the result is
  normalised by a softmax and then multiplied with the values
  (page "FlashAttention 4: Γρηγορότερη και Αποδοτική σε Μνήμη Προσοχή για LLMs",
  section "Εισαγωγή").  The scores are scaled before any modification:
  s_ij = scale * <q_i, k_j>.
* The score modifications and masks are the FlexAttention variants named on the page
  "PyTorch's FlexAttention mit FlashAttention-4 ist ein Game-Changer" (intro
  paragraph listing ALiBi, sliding window, document masking and soft-capping) and
  causal attention (same page, section "Leistung und Validierung").
* The output keeps, per query row, only the running maximum and sum of the softmax
  (page "FlashAttention 4 ...", section "Γιατί οι πυρήνες προσοχής ..."); the oracle
  returns the log-sum-exp built from those two, LSE_i = m_i + ln(l_i), in natural log.

Readings taken where the pages are silent:
* Layout [B, H, S, D].  Causal alignment is bottom-right: query row i sits at key
  position i' = i + (Sk - Sq).
* Sliding window W counts the diagonal: causal+window keeps 0 <= i' - j < W; window
  without causal keeps |i' - j| < W.
* Soft-capping acts on the scaled score: s <- c * tanh(s / c); ALiBi is added after it:
  s <- s + slope_h * (j - i').
* Document masking keeps a pair iff doc[b, i] == doc[b, j] (requires Sq == Sk).
* A row with no visible key has O = 0 and LSE = -inf.

The computation is the two-pass softmax of the definition — max, exponentials, sum,
normalise, multiply — with no tiling and no online rescaling.
"""
from __future__ import annotations

import numpy as np

MASK_CAUSAL = 1
MASK_WINDOW = 2
MASK_DOC = 4


def visible_mask(rows: np.ndarray, Sq: int, Sk: int, mask_kind: int, window: int,
                 doc_row: np.ndarray | None) -> np.ndarray:
    """Boolean [len(rows), Sk]: True where key j is visible to query row i."""
    rows = np.asarray(rows, dtype=np.int64)
    ip = rows[:, None] + (Sk - Sq)          # bottom-right aligned query position
    j = np.arange(Sk, dtype=np.int64)[None, :]
    vis = np.ones((rows.shape[0], Sk), dtype=bool)
    if mask_kind & MASK_CAUSAL:
        vis &= j <= ip
    if mask_kind & MASK_WINDOW:
        if mask_kind & MASK_CAUSAL:
            vis &= (ip - j) < window
        else:
            vis &= np.abs(ip - j) < window
    if mask_kind & MASK_DOC:
        if doc_row is None:
            raise ValueError("document mask needs doc ids")
        d = np.asarray(doc_row)
        vis &= d[rows][:, None] == d[None, :Sk]
    return vis


def modified_scores(q_rows: np.ndarray, k: np.ndarray, scale: float, rows: np.ndarray,
                    Sq: int, Sk: int, softcap: float, slope: float | None) -> np.ndarray:
    """s = scale * q k^T, then soft-capping, then ALiBi, all in float64."""
    s = (q_rows.astype(np.float64) @ k.astype(np.float64).T) * float(scale)
    if softcap and softcap > 0:
        c = float(softcap)
        s = c * np.tanh(s / c)
    if slope is not None:
        ip = np.asarray(rows, dtype=np.int64)[:, None] + (Sk - Sq)
        j = np.arange(Sk, dtype=np.int64)[None, :]
        s = s + float(slope) * (j - ip).astype(np.float64)
    return s


def softmax_rows(s: np.ndarray, vis: np.ndarray):
    """Two-pass softmax over the visible entries of each row.

    Returns (P, m, l): P the normalised weights (0 where masked), m the row maximum of
    the visible scores, l the sum of exp(s - m).  Rows with nothing visible get P = 0,
    m = -inf, l = 0."""
    sm = np.where(vis, s, -np.inf)
    m = sm.max(axis=1)
    any_vis = vis.any(axis=1)
    m_safe = np.where(any_vis, m, 0.0)
    e = np.where(vis, np.exp(sm - m_safe[:, None]), 0.0)
    l = e.sum(axis=1)
    P = np.divide(e, l[:, None], out=np.zeros_like(e), where=l[:, None] > 0)
    return P, np.where(any_vis, m, -np.inf), l


def attention_fwd(q, k, v, scale: float, mask_kind: int = 0, window: int = 0,
                  softcap: float = 0.0, alibi_slopes=None, doc_ids=None, rows=None,
                  chunk: int = 512):
    """fp64 attention forward.

    q: [B,H,Sq,D], k, v: [B,Hkv,Sk,D] (any float dtype; converted exactly to float64).
    Hkv divides H: query head h reads key/value head h // (H // Hkv) (grouped-query
    attention; Hkv = 1 is multi-query attention, Hkv = H plain multi-head attention).
    alibi_slopes: None or [H].  doc_ids: None or int [B, S] (Sq == Sk).
    rows: None for every query row, else a 1-D array of query rows to evaluate (rows are
    independent given the full K and V, so a subset is exact for those rows).
    Returns (O [B,H,R,D] float64, LSE [B,H,R] float64) with R = Sq or len(rows).
    """
    q = _f64(q)
    k = _f64(k)
    v = _f64(v)
    B, H, Sq, D = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    if H % Hkv != 0:
        raise ValueError("the number of key/value heads must divide the number of query heads")
    group = H // Hkv
    if mask_kind & MASK_DOC and Sq != Sk:
        raise ValueError("document mask needs Sq == Sk")
    rows = np.arange(Sq, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    slopes = None if alibi_slopes is None else _f64(alibi_slopes).reshape(-1)
    docs = None if doc_ids is None else np.asarray(
        doc_ids.cpu().numpy() if hasattr(doc_ids, "cpu") else doc_ids)
    R = rows.shape[0]
    O = np.zeros((B, H, R, D), dtype=np.float64)
    LSE = np.full((B, H, R), -np.inf, dtype=np.float64)
    for b in range(B):
        doc_row = None if docs is None else docs[b]
        for r0 in range(0, R, chunk):
            rr = rows[r0:r0 + chunk]
            vis = visible_mask(rr, Sq, Sk, mask_kind, window, doc_row)
            for h in range(H):
                slope = None if slopes is None else slopes[h]
                hk = h // group
                s = modified_scores(q[b, h, rr], k[b, hk], scale, rr, Sq, Sk, softcap, slope)
                P, m, l = softmax_rows(s, vis)
                O[b, h, r0:r0 + len(rr)] = P @ v[b, hk]
                with np.errstate(divide="ignore"):
                    LSE[b, h, r0:r0 + len(rr)] = np.where(l > 0, m + np.log(l), -np.inf)
    return O, LSE


def attention_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, scale: float, mask_kind: int = 0,
                         window: int = 0, softcap: float = 0.0, alibi_slopes=None):
    """fp64 attention over packed variable-length sequences.

    Sequence s holds query tokens cu_seqlens_q[s] .. cu_seqlens_q[s+1]-1 and key tokens
    cu_seqlens_k[s] .. cu_seqlens_k[s+1]-1; it attends only within itself, exactly as a
    separate batch entry of its own lengths would (masks, causal alignment and ALiBi
    positions are per sequence).  Token-major layout: q [Tq, H, D], k, v [Tk, Hkv, D].
    Returns (O [Tq, H, D], LSE [H, Tq]) in float64; tokens of no sequence stay O = 0,
    LSE = -inf."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    cq = np.asarray(cu_seqlens_q, dtype=np.int64).reshape(-1)
    ck = np.asarray(cu_seqlens_k, dtype=np.int64).reshape(-1)
    Tq, H, D = q.shape
    O = np.zeros((Tq, H, D), dtype=np.float64)
    LSE = np.full((H, Tq), -np.inf, dtype=np.float64)
    for s in range(len(cq) - 1):
        q0, q1, k0, k1 = cq[s], cq[s + 1], ck[s], ck[s + 1]
        if q1 <= q0:
            continue
        if k1 <= k0:
            continue
        qs = q[q0:q1].transpose(1, 0, 2)[None]
        ks = k[k0:k1].transpose(1, 0, 2)[None]
        vs = v[k0:k1].transpose(1, 0, 2)[None]
        o, lse = attention_fwd(qs, ks, vs, scale, mask_kind, window, softcap, alibi_slopes)
        O[q0:q1] = o[0].transpose(1, 0, 2)
        LSE[:, q0:q1] = lse[0]
    return O, LSE


def visible_pair_count(Sq: int, Sk: int, mask_kind: int, window: int, doc_row=None,
                       chunk: int = 2048) -> int:
    """Number of visible (i, j) pairs for one (b, h), by brute force over the mask."""
    total = 0
    for r0 in range(0, Sq, chunk):
        rr = np.arange(r0, min(Sq, r0 + chunk))
        total += int(visible_mask(rr, Sq, Sk, mask_kind, window, doc_row).sum())
    return total


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):
        return x.detach().cpu().to(dtype=__import__("torch").float64).numpy()
    return np.asarray(x, dtype=np.float64)
