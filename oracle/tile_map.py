"""Block-sparse tile map by brute force — oracle (test infrastructure only).

FlexAttention skips blocks that the mask removes entirely (page "PyTorch's
FlexAttention mit FlashAttention-4 ist ein Game-Changer", section "Aktuelle
Einschränkungen", on block sparsity).  The oracle classifies every (query block, key
tile) pair from the element mask itself:

* EMPTY (0)   no visible pair among the valid rows (i < Sq) and valid keys (j < Sk);
* FULL (2)    every key column of the tile is valid (j < Sk) and visible to every valid row;
* PARTIAL (1) anything else.

Geometry and encoding (the C-ABI's tile-map format): query blocks of 256 rows, each made
of two 128-row query tiles (tile 0 = rows 0..127 of the block, tile 1 = rows 128..255);
key tiles of 128 columns.  For each (b, query block) the map lists, in increasing order,
the key tiles for which at least one of the two query tiles is not EMPTY, as

    entry = kt | (class_tile0 << 24) | (class_tile1 << 26)

and ``counts[b, qb]`` is the length of that list.  A query tile with no valid row is
EMPTY everywhere.
"""
from __future__ import annotations

import numpy as np

from .attention import visible_mask

EMPTY, PARTIAL, FULL = 0, 1, 2
BLOCK_Q = 256
TILE_Q = 128
TILE_K = 128


def classify(vis: np.ndarray, n_valid_cols: int) -> int:
    """Class of one (query tile, key tile) from its visibility matrix over valid rows."""
    if vis.size == 0 or not vis.any():
        return EMPTY
    if n_valid_cols == TILE_K and vis.all():
        return FULL
    return PARTIAL


def tile_map(B: int, Sq: int, Sk: int, mask_kind: int, window: int, doc_ids=None):
    """Returns (counts int32 [B, nqb], entries uint32 [B, nqb, nkt])."""
    nqb = (Sq + BLOCK_Q - 1) // BLOCK_Q
    nkt = (Sk + TILE_K - 1) // TILE_K
    docs = None
    if doc_ids is not None:
        docs = np.asarray(doc_ids.cpu().numpy() if hasattr(doc_ids, "cpu") else doc_ids)
    counts = np.zeros((B, nqb), dtype=np.int32)
    entries = np.zeros((B, nqb, nkt), dtype=np.uint32)
    for b in range(B):
        doc_row = None if docs is None else docs[b]
        for qb in range(nqb):
            cls_rows = []
            for t in range(2):
                r0 = qb * BLOCK_Q + t * TILE_Q
                rows = np.arange(r0, min(Sq, r0 + TILE_Q))
                vis = visible_mask(rows, Sq, Sk, mask_kind, window, doc_row) if rows.size \
                    else np.zeros((0, Sk), dtype=bool)
                per_kt = []
                for kt in range(nkt):
                    c0, c1 = kt * TILE_K, min(Sk, (kt + 1) * TILE_K)
                    per_kt.append(classify(vis[:, c0:c1], c1 - c0))
                cls_rows.append(per_kt)
            n = 0
            for kt in range(nkt):
                c0, c1 = cls_rows[0][kt], cls_rows[1][kt]
                if c0 == EMPTY and c1 == EMPTY:
                    continue
                entries[b, qb, n] = kt | (c0 << 24) | (c1 << 26)
                n += 1
            counts[b, qb] = n
    return counts, entries
