"""GPU parity of attn_fwd_pair (the forward on 2-CTA clusters, tcgen05 cta_group::2) against
the fp64 oracle, with the same gates as attn_fwd.

The cases cover what is particular to the pair split: the odd CTA's query rows past Sq, the
odd CTA's half of a key tile past Sk (its K rows are TMA zero fill), items with one key tile,
every mask and score modification, unsorted document ids (per-element test on a half tile),
grouped-query heads, the rescale threshold (scores far from zero), a full-size sampled
configuration, run-to-run bitwise determinism and the rejection of other head dimensions."""
import math

import numpy as np
import pytest
import torch

from attn_workloads import (MASK_CAUSAL, MASK_DOC, MASK_NONE, MASK_WINDOW, WORKLOADS, alibi_slopes,
                            doc_ids_from_lengths, make_doc_ids, make_qkv, sample_rows)
from tests.gpu_helpers import compare, oracle_eav, to_dev

pytestmark = pytest.mark.gpu


def _run(B, H, Sq, Sk, mask=MASK_NONE, window=0, softcap=0.0, alibi=False, doc=None, seed=0, q_mul=1.0, Hkv=None):
    import tiled_attention_14_b200 as ta
    D = 128
    q, k, v = make_qkv(B, H, Sq, Sk, D, seed=seed, q_mul=q_mul, Hkv=Hkv)
    sl = alibi_slopes(H) if alibi else None
    scale = 1.0 / math.sqrt(D)
    qd, kd, vd, sld, docd = to_dev(q, k, v, sl, doc)
    o, lse = ta.attn_fwd_pair(qd, kd, vd, scale=scale, mask_kind=mask, window=window, softcap=softcap,
                              alibi_slopes=sld, doc_ids=docd)
    torch.cuda.synchronize()
    assert ta.attn_get_status() == 0
    O, L, E = oracle_eav(q, k, v, scale, mask, window, softcap, sl, doc)
    return compare(o, lse, O, L, eav=E)


@pytest.mark.parametrize("Sq,Sk", [(256, 256), (300, 300), (640, 384), (130, 700), (1, 129), (777, 1), (200, 64)])
def test_no_mask_shapes(Sq, Sk):
    _run(2, 3, Sq, Sk, seed=Sq + Sk)


@pytest.mark.parametrize("Sq,Sk", [(640, 640), (300, 300), (200, 520), (520, 200), (129, 129)])
def test_causal_shapes(Sq, Sk):
    _run(2, 2, Sq, Sk, MASK_CAUSAL, seed=Sq * 3 + Sk)


@pytest.mark.parametrize("W,causal", [(1, True), (100, True), (300, False), (5000, True)])
def test_window(W, causal):
    _run(1, 2, 900, 900, MASK_WINDOW | (MASK_CAUSAL if causal else 0), window=W, seed=W)


@pytest.mark.parametrize("causal", [True, False])
def test_alibi_and_softcap(causal):
    m = MASK_CAUSAL if causal else MASK_NONE
    _run(1, 4, 700, 700, m, alibi=True, seed=31)
    _run(1, 2, 520, 520, m, softcap=30.0, seed=32, q_mul=8.0)
    _run(1, 2, 600, 600, m, softcap=50.0, alibi=True, seed=33)


@pytest.mark.parametrize("lens", [[300, 129, 1, 450, 144], [1] * 7 + [993]])
def test_document_mask(lens):
    S = sum(lens)
    doc = torch.from_numpy(np.stack([doc_ids_from_lengths(lens), doc_ids_from_lengths(lens[::-1])]))
    _run(2, 2, S, S, MASK_DOC | MASK_CAUSAL, doc=doc, seed=S)


def test_document_mask_unsorted_ids():
    rng = np.random.default_rng(3)
    S = 650
    doc = torch.from_numpy(rng.integers(0, 3, size=(1, S)).astype(np.int32))
    _run(1, 2, S, S, MASK_DOC, doc=doc, seed=11)


@pytest.mark.parametrize("H,Hkv", [(8, 2), (4, 1)])
def test_grouped_heads(H, Hkv):
    _run(2, H, 520, 520, MASK_CAUSAL, seed=H + Hkv, Hkv=Hkv)


def test_large_scale_values():
    """Scores far from zero exercise the rescale threshold, and with it the wait for the
    previous P V that the pair kernel takes from the next S's completion."""
    _run(1, 2, 1024, 1024, MASK_NONE, seed=12, q_mul=6.0)
    _run(1, 2, 1024, 1024, MASK_CAUSAL, seed=13, q_mul=6.0)


def test_full_size_sampled_rows_causal():
    import tiled_attention_14_b200 as ta
    w = WORKLOADS["causal"]
    q, k, v = make_qkv(w.B, w.H, w.Sq, w.Sk, w.D, seed=0)
    rows = sample_rows(w.Sq, 24, seed=1)
    qd, kd, vd = to_dev(q, k, v)
    o, lse = ta.attn_fwd_pair(qd, kd, vd, scale=w.scale, mask_kind=w.mask_kind)
    torch.cuda.synchronize()
    assert ta.attn_get_status() == 0
    O, L, E = oracle_eav(q, k, v, w.scale, w.mask_kind, rows=rows)
    compare(o, lse, O, L, rows=rows, eav=E)


def test_deterministic():
    import tiled_attention_14_b200 as ta
    q, k, v = to_dev(*make_qkv(2, 4, 1000, 1000, 128, seed=21))
    o1, l1 = ta.attn_fwd_pair(q, k, v, mask_kind=MASK_CAUSAL)
    o2, l2 = ta.attn_fwd_pair(q, k, v, mask_kind=MASK_CAUSAL)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_other_head_dims_rejected():
    import tiled_attention_14_b200 as ta
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        ta.attn_fwd_pair(q, q, q)
