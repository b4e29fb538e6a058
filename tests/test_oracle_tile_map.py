"""Pins for the oracle's block-sparse tile map (CPU only): closed forms for the causal,
window and ragged-edge cases, and coverage invariants for document masks."""
import numpy as np
import pytest

from oracle.attention import visible_mask
from oracle.tile_map import EMPTY, FULL, PARTIAL, tile_map
from attn_workloads import MASK_CAUSAL, MASK_DOC, MASK_NONE, MASK_WINDOW, doc_ids_from_lengths


def _decode(counts, entries, b, qb):
    out = {}
    for e in entries[b, qb, :counts[b, qb]]:
        e = int(e)
        out[e & 0xFFFFFF] = ((e >> 24) & 3, (e >> 26) & 3)
    return out


def test_no_mask_ragged_edge():
    counts, entries = tile_map(1, 300, 300, MASK_NONE, 0)
    assert counts.tolist() == [[3, 3]]
    m = _decode(counts, entries, 0, 0)
    assert m == {0: (FULL, FULL), 1: (FULL, FULL), 2: (PARTIAL, PARTIAL)}
    m = _decode(counts, entries, 0, 1)          # rows 256..299: tile 1 has no valid row
    assert m == {0: (FULL, EMPTY), 1: (FULL, EMPTY), 2: (PARTIAL, EMPTY)}


def test_causal_closed_form():
    S = 1024
    counts, entries = tile_map(1, S, S, MASK_CAUSAL, 0)
    for qb in range(S // 256):
        m = _decode(counts, entries, 0, qb)
        assert sorted(m) == list(range(2 * qb + 2))
        for kt, (c0, c1) in m.items():
            assert c0 == (FULL if kt < 2 * qb else PARTIAL if kt == 2 * qb else EMPTY)
            assert c1 == (FULL if kt < 2 * qb + 1 else PARTIAL)


def test_causal_window_closed_form():
    S, W = 2048, 300
    counts, entries = tile_map(1, S, S, MASK_CAUSAL | MASK_WINDOW, W)
    for qb in range(S // 256):
        m = _decode(counts, entries, 0, qb)
        for t in range(2):
            r0 = qb * 256 + t * 128
            r1 = r0 + 127
            lo_key, hi_key = max(0, r0 - W + 1), r1
            for kt in range(S // 128):
                c0, c1 = kt * 128, kt * 128 + 127
                cls = m.get(kt, (EMPTY, EMPTY))[t]
                if c1 < lo_key or c0 > hi_key:
                    assert cls == EMPTY
                elif c1 <= r0 and c0 >= r1 - W + 1:
                    assert cls == FULL
                else:
                    assert cls == PARTIAL


@pytest.mark.parametrize("mask", [MASK_DOC, MASK_DOC | MASK_CAUSAL])
def test_document_map_covers_every_visible_pair(mask):
    lens = [100, 300, 37, 200, 131]
    S = sum(lens)
    doc = doc_ids_from_lengths(lens)[None]
    counts, entries = tile_map(1, S, S, mask, 0, doc)
    vis = visible_mask(np.arange(S), S, S, mask, 0, doc[0])
    nkt = (S + 127) // 128
    for qb in range((S + 255) // 256):
        m = _decode(counts, entries, 0, qb)
        for t in range(2):
            r0 = qb * 256 + t * 128
            rows = slice(r0, min(S, r0 + 128))
            for kt in range(nkt):
                blk = vis[rows, kt * 128:(kt + 1) * 128]
                cls = m.get(kt, (EMPTY, EMPTY))[t]
                if blk.size == 0 or not blk.any():
                    assert cls == EMPTY
                elif blk.all() and blk.shape[1] == 128:
                    assert cls == FULL
                else:
                    assert cls == PARTIAL
        # listed tiles are increasing
        ks = [int(e) & 0xFFFFFF for e in entries[0, qb, :counts[0, qb]]]
        assert ks == sorted(ks)


def test_single_document_is_dense():
    S = 512
    doc = np.zeros((2, S), dtype=np.int32)
    c1, e1 = tile_map(2, S, S, MASK_DOC, 0, doc)
    c0, e0 = tile_map(2, S, S, MASK_NONE, 0)
    np.testing.assert_array_equal(c1, c0)
    np.testing.assert_array_equal(e1, e0)
