"""GPU parity of grouped-query heads (attn_fwd_gqa) and packed variable-length sequences
(attn_fwd_varlen) against the fp64 oracle, through the C-ABI.  Every output element is
compared at sizes that span several tiles and ragged tails; the BF16 gate of the plain
path applies (|dO| <= 1e-2 + 2^-8 (|O| + E_p|v|) per element, max|dLSE| <= 1e-3)."""
import math

import numpy as np
import pytest
import torch

from attn_workloads import (MASK_CAUSAL, MASK_DOC, MASK_NONE, MASK_WINDOW, WORKLOADS, alibi_slopes,
                            doc_ids_from_lengths, make_qkv, varlen_cu_seqlens)
from oracle.attention import attention_fwd, attention_fwd_varlen
from tests.gpu_helpers import compare, oracle_eav, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("H,Hkv", [(16, 16), (16, 4), (16, 1)])
@pytest.mark.parametrize("mask", [MASK_NONE, MASK_CAUSAL])
@pytest.mark.parametrize("D", [64, 128])
def test_gqa(H, Hkv, mask, D):
    import tiled_attention_14_b200 as ta
    B, S = 2, 520
    q, k, v = make_qkv(B, H, S, S, D, seed=H + Hkv + D, Hkv=Hkv)
    qd, kd, vd = to_dev(q, k, v)
    o, lse = ta.attn_fwd(qd, kd, vd, mask_kind=mask)
    torch.cuda.synchronize()
    assert ta.attn_get_status() == 0
    O, L, E = oracle_eav(q, k, v, 1.0 / math.sqrt(D), mask)
    compare(o, lse, O, L, eav=E)


def test_gqa_with_score_mods_and_masks():
    import tiled_attention_14_b200 as ta
    B, H, Hkv, S, D = 1, 8, 2, 700, 128
    q, k, v = make_qkv(B, H, S, S, D, seed=3, Hkv=Hkv)
    sl = alibi_slopes(H)
    qd, kd, vd, sld = to_dev(q, k, v, sl)
    scale = 1.0 / math.sqrt(D)
    cases = [dict(mask_kind=MASK_CAUSAL | MASK_WINDOW, window=200, alibi=True),
             dict(mask_kind=MASK_NONE, softcap=30.0),
             dict(mask_kind=MASK_WINDOW, window=90)]
    for c in cases:
        o, lse = ta.attn_fwd(qd, kd, vd, mask_kind=c["mask_kind"], window=c.get("window", 0),
                             softcap=c.get("softcap", 0.0), alibi_slopes=sld if c.get("alibi") else None)
        torch.cuda.synchronize()
        assert ta.attn_get_status() == 0
        O, L, E = oracle_eav(q, k, v, scale, c["mask_kind"], c.get("window", 0), c.get("softcap", 0.0),
                             sl if c.get("alibi") else None)
        compare(o, lse, O, L, eav=E)


def test_gqa_document_mask():
    import tiled_attention_14_b200 as ta
    lens = [300, 129, 1, 450, 144]
    S = sum(lens)
    doc = torch.from_numpy(np.stack([doc_ids_from_lengths(lens), doc_ids_from_lengths(lens[::-1])]))
    q, k, v = make_qkv(2, 4, S, S, 128, seed=9, Hkv=1)
    qd, kd, vd, docd = to_dev(q, k, v, doc)
    o, lse = ta.attn_fwd(qd, kd, vd, mask_kind=MASK_DOC | MASK_CAUSAL, doc_ids=docd)
    torch.cuda.synchronize()
    assert ta.attn_get_status() == 0
    O, L, E = oracle_eav(q, k, v, 1.0 / math.sqrt(128), MASK_DOC | MASK_CAUSAL, 0, 0.0, None, doc)
    compare(o, lse, O, L, eav=E)


def _cmp_packed(o, lse, O, L, E):
    """compare() on the packed layout: o [T,H,D] and lse [H,T] become [1,H,T,D] / [1,H,T]."""
    return compare(o.permute(1, 0, 2)[None], lse[None], O.transpose(1, 0, 2)[None], L[None],
                   eav=E.transpose(1, 0, 2)[None])


def _varlen_oracle(q, k, v, cq, ck, scale, *args):
    """(O, LSE, E_p|v|) of packed sequences."""
    O, L = attention_fwd_varlen(q, k, v, cq, ck, scale, *args)
    E, _ = attention_fwd_varlen(q, k, v.abs(), cq, ck, scale, *args)
    return O, L, E


def _varlen_inputs(lq, lk, H, Hkv, D, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(sum(lq), H, D, generator=g).to(torch.bfloat16)
    k = torch.randn(sum(lk), Hkv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(sum(lk), Hkv, D, generator=g).to(torch.bfloat16)
    cq = torch.tensor(np.concatenate([[0], np.cumsum(lq)]), dtype=torch.int32)
    ck = torch.tensor(np.concatenate([[0], np.cumsum(lk)]), dtype=torch.int32)
    return q, k, v, cq, ck


def _varlen_case(lq, lk, H, Hkv, D, mask=MASK_NONE, window=0, softcap=0.0, alibi=False, seed=0):
    import tiled_attention_14_b200 as ta
    q, k, v, cq, ck = _varlen_inputs(lq, lk, H, Hkv, D, seed)
    sl = alibi_slopes(H) if alibi else None
    qd, kd, vd, cqd, ckd, sld = to_dev(q, k, v, cq, ck, sl)
    o, lse = ta.attn_fwd_varlen(qd, kd, vd, cqd, ckd, max(lq), max(lk), mask_kind=mask, window=window,
                                softcap=softcap, alibi_slopes=sld)
    torch.cuda.synchronize()
    assert ta.attn_get_status() == 0
    O, L, E = _varlen_oracle(q, k, v, cq.numpy(), ck.numpy(), 1.0 / math.sqrt(D), mask, window, softcap,
                             None if sl is None else sl.numpy())
    return _cmp_packed(o, lse, O, L, E)


@pytest.mark.parametrize("mask", [MASK_NONE, MASK_CAUSAL])
@pytest.mark.parametrize("D", [64, 128])
def test_varlen_equal_lengths(mask, D):
    lens = [1, 127, 128, 129, 300, 1000, 45]
    _varlen_case(lens, lens, 8, 2, D, mask, seed=D + mask)


@pytest.mark.parametrize("mask,window", [(MASK_CAUSAL, 0), (MASK_CAUSAL | MASK_WINDOW, 100), (MASK_WINDOW, 64),
                                         (MASK_NONE, 0)])
def test_varlen_unequal_lengths(mask, window):
    """Sq != Sk per sequence (bottom-right alignment), an empty query sequence and a
    sequence without keys."""
    lq = [200, 0, 513, 77, 130, 5]
    lk = [350, 40, 257, 77, 0, 600]
    _varlen_case(lq, lk, 4, 4, 128, mask, window, seed=window + 1)


def test_varlen_score_mods():
    lens = [260, 700, 33]
    _varlen_case(lens, lens, 4, 1, 128, MASK_CAUSAL, alibi=True, seed=5)
    _varlen_case(lens, lens, 4, 2, 128, MASK_NONE, softcap=20.0, seed=6)


def test_varlen_benchmark_packing_sampled():
    """The packed workload of the benchmark (document lengths of config 3d) against the
    oracle on a few whole sequences."""
    import tiled_attention_14_b200 as ta
    w = WORKLOADS["varlen"]
    cu = varlen_cu_seqlens(w.B, w.Sq)
    T = int(cu[-1])
    lens = np.diff(cu.numpy())
    g = torch.Generator().manual_seed(0)
    q = torch.randn(T, w.H, w.D, generator=g).to(torch.bfloat16)
    k = torch.randn(T, w.H, w.D, generator=g).to(torch.bfloat16)
    v = torch.randn(T, w.H, w.D, generator=g).to(torch.bfloat16)
    qd, kd, vd, cud = to_dev(q, k, v, cu)
    o, lse = ta.attn_fwd_varlen(qd, kd, vd, cud, cud, int(lens.max()), int(lens.max()))
    torch.cuda.synchronize()
    assert ta.attn_get_status() == 0
    for s in (0, len(lens) // 2, len(lens) - 1):
        a, b = int(cu[s]), int(cu[s + 1])
        sub = torch.tensor([0, b - a], dtype=torch.int32)
        O, L, E = _varlen_oracle(q[a:b], k[a:b], v[a:b], sub.numpy(), sub.numpy(), w.scale)
        _cmp_packed(o[a:b], lse[:, a:b], O, L, E)


def test_varlen_offsets_out_of_range_are_reported():
    """A sequence longer than the stated maximum is skipped and reported; the others are
    computed (the kernel checks every sequence's bounds before it loads anything)."""
    import tiled_attention_14_b200 as ta
    lq = [100, 300, 50]
    q, k, v, cq, ck = _varlen_inputs(lq, lq, 2, 2, 128, seed=1)
    qd, kd, vd, cqd, ckd = to_dev(q, k, v, cq, ck)
    o = torch.full((sum(lq), 2, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((2, sum(lq)), 7.0, device="cuda")
    ta.attn_fwd_varlen(qd, kd, vd, cqd, ckd, 256, 256, o=o, lse=lse)   # sequence 1 is longer than 256
    torch.cuda.synchronize()
    assert ta.attn_get_status() == ta._lib.ATTN_ERR_INVALID
    assert torch.all(o[100:400] == 7.0) and torch.all(lse[:, 100:400] == 7.0)
    O, L, E = _varlen_oracle(q, k, v, cq.numpy(), ck.numpy(), 1.0 / math.sqrt(128))
    keep = np.r_[0:100, 400:450]
    kt = torch.from_numpy(keep).cuda()
    _cmp_packed(o[kt], lse[:, kt], O[keep], L[:, keep], E[keep])
    assert ta.attn_get_status() == 0
