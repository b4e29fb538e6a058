"""GPU parity of the BF16 attention forward (through the C-ABI) against the fp64 oracle.

Small cases compare every output element; they span several 128-row / 128-column tiles
and ragged tails.  Full-size benchmark shapes compare sampled query rows, which the
oracle computes exactly from the full K and V."""
import math

import numpy as np
import pytest
import torch

from attn_workloads import (MASK_CAUSAL, MASK_DOC, MASK_NONE, MASK_WINDOW, WORKLOADS, alibi_slopes,
                            doc_ids_from_lengths, make_doc_ids, make_qkv, sample_rows)
from tests.gpu_helpers import compare, oracle_eav, to_dev

pytestmark = pytest.mark.gpu


def _run(B, H, Sq, Sk, D, mask=MASK_NONE, window=0, softcap=0.0, alibi=False, doc=None, seed=0,
         q_mul=1.0, scale=None):
    import tiled_attention_14_b200 as ta
    q, k, v = make_qkv(B, H, Sq, Sk, D, seed=seed, q_mul=q_mul)
    sl = alibi_slopes(H) if alibi else None
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    qd, kd, vd, sld, docd = to_dev(q, k, v, sl, doc)
    o, lse = ta.attn_fwd(qd, kd, vd, scale=scale, mask_kind=mask, window=window, softcap=softcap,
                         alibi_slopes=sld, doc_ids=docd)
    torch.cuda.synchronize()
    assert ta.attn_get_status() == 0
    O, L, E = oracle_eav(q, k, v, scale, mask, window, softcap, sl, doc)
    return compare(o, lse, O, L, eav=E)


def test_tiny_config():
    w = WORKLOADS["tiny"]
    _run(w.B, w.H, w.Sq, w.Sk, w.D)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Sq,Sk", [(256, 256), (300, 300), (640, 384), (130, 700), (1, 129), (777, 1)])
def test_no_mask_shapes(D, Sq, Sk):
    _run(1, 3, Sq, Sk, D, seed=Sq + Sk)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Sq,Sk", [(640, 640), (300, 300), (200, 520), (520, 200), (129, 129)])
def test_causal_shapes(D, Sq, Sk):
    _run(2, 2, Sq, Sk, D, MASK_CAUSAL, seed=Sq * 3 + Sk)


@pytest.mark.parametrize("W", [1, 100, 128, 300, 5000])
@pytest.mark.parametrize("causal", [True, False])
def test_window(W, causal):
    mask = MASK_WINDOW | (MASK_CAUSAL if causal else 0)
    _run(1, 2, 700, 700, 128, mask, window=W, seed=W)


def test_window_ragged_rectangular():
    _run(1, 2, 333, 901, 128, MASK_WINDOW | MASK_CAUSAL, window=200, seed=4)
    _run(1, 2, 901, 333, 64, MASK_WINDOW, window=77, seed=5)


@pytest.mark.parametrize("causal", [True, False])
def test_alibi(causal):
    _run(1, 4, 600, 600, 128, MASK_CAUSAL if causal else MASK_NONE, alibi=True, seed=6)


@pytest.mark.parametrize("q_mul", [1.0, 8.0])
def test_softcap(q_mul):
    _run(1, 2, 520, 520, 128, MASK_NONE, softcap=50.0, seed=7, q_mul=q_mul)
    _run(1, 2, 300, 300, 64, MASK_CAUSAL, softcap=5.0, seed=8, q_mul=q_mul)


def test_softcap_with_alibi_causal():
    _run(1, 2, 400, 400, 128, MASK_CAUSAL, softcap=20.0, alibi=True, seed=9)


@pytest.mark.parametrize("lens", [[300, 129, 1, 450, 144], [1000], [1] * 7 + [993], [128, 128, 256, 488]])
@pytest.mark.parametrize("causal", [False, True])
def test_document_mask(lens, causal):
    S = sum(lens)
    doc = torch.from_numpy(np.stack([doc_ids_from_lengths(lens), doc_ids_from_lengths(lens[::-1])]))
    _run(2, 2, S, S, 128, MASK_DOC | (MASK_CAUSAL if causal else 0), doc=doc, seed=S)


def test_document_mask_unsorted_ids():
    """Document ids that are not a running index (ids repeat in separate runs)."""
    rng = np.random.default_rng(3)
    S = 650
    doc = torch.from_numpy(rng.integers(0, 3, size=(1, S)).astype(np.int32))
    _run(1, 2, S, S, 128, MASK_DOC, doc=doc, seed=11)


def test_large_scale_values():
    """Scores far from zero exercise the rescale threshold (max moves by > 8 in log2)."""
    _run(1, 2, 1024, 1024, 128, MASK_NONE, seed=12, q_mul=6.0)
    _run(1, 2, 1024, 1024, 128, MASK_CAUSAL, seed=13, q_mul=6.0)


def test_bh_below_sm_count_and_many_items():
    _run(1, 1, 4096, 4096, 64, MASK_CAUSAL, seed=14)


def _sampled(w, n_random=24, q_mul=1.0):
    import tiled_attention_14_b200 as ta
    q, k, v = make_qkv(w.B, w.H, w.Sq, w.Sk, w.D, seed=0)
    sl = alibi_slopes(w.H) if w.alibi else None
    doc = make_doc_ids(w.B, w.Sq) if w.doc else None
    extra = []
    if doc is not None:
        d = doc[0].numpy()
        starts = np.flatnonzero(np.diff(d)) + 1
        extra = list(starts) + list(starts - 1)
    rows = sample_rows(w.Sq, n_random, seed=1, extra=extra)
    qd, kd, vd, sld, docd = to_dev(q, k, v, sl, doc)
    o, lse = ta.attn_fwd(qd, kd, vd, scale=w.scale, mask_kind=w.mask_kind, window=w.window,
                         softcap=w.softcap, alibi_slopes=sld, doc_ids=docd)
    torch.cuda.synchronize()
    assert ta.attn_get_status() == 0
    O, L, E = oracle_eav(q, k, v, w.scale, w.mask_kind, w.window, w.softcap, sl, doc, rows=rows)
    return compare(o, lse, O, L, rows=rows, eav=E)


@pytest.mark.parametrize("name", ["causal", "window", "alibi", "softcap", "doc", "long"])
def test_full_size_sampled_rows(name):
    _sampled(WORKLOADS[name])


def test_deterministic():
    import tiled_attention_14_b200 as ta
    q, k, v = to_dev(*make_qkv(2, 4, 1000, 1000, 128, seed=21))
    o1, l1 = ta.attn_fwd(q, k, v, mask_kind=MASK_CAUSAL)
    o2, l2 = ta.attn_fwd(q, k, v, mask_kind=MASK_CAUSAL)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("mask,window,lens", [
    (MASK_CAUSAL, 0, None), (MASK_CAUSAL | MASK_WINDOW, 200, None), (MASK_WINDOW, 150, None),
    (MASK_DOC, 0, [300, 129, 1, 450, 144]), (MASK_NONE, 0, None)])
def test_tile_skip_identity(mask, window, lens):
    """Skipping fully masked tiles equals visiting every tile as PARTIAL, bit for bit."""
    import tiled_attention_14_b200 as ta
    S = 1024 if lens is None else sum(lens)
    doc = None if lens is None else torch.from_numpy(doc_ids_from_lengths(lens)[None].repeat(2, 0))
    q, k, v, docd = to_dev(*make_qkv(2, 2, S, S, 128, seed=22), doc)
    o1, l1 = ta.attn_fwd(q, k, v, mask_kind=mask, window=window, doc_ids=docd)
    nqb, nkt = (S + 255) // 256, (S + 127) // 128
    counts = torch.full((2, nqb), nkt, dtype=torch.int32, device="cuda")
    ent = torch.arange(nkt, dtype=torch.int64) | (1 << 24) | (1 << 26)
    entries = ent.to(torch.int32).repeat(2, nqb, 1).cuda().contiguous()
    o2, l2 = ta.attn_fwd_with_map(q, k, v, counts, entries, mask_kind=mask, window=window, doc_ids=docd)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    assert torch.equal(l1, l2)
