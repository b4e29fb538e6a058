"""Pins for the oracle's grouped-query heads and packed variable-length sequences (CPU).

Grouped-query / multi-query attention: query heads share key/value heads (page
"FlashAttention 4: ...", section "Συμβατότητα και τρέχουσα κατάσταση", which names GQA and
variable-length batches without padding as missing from FA4).  The oracle's mapping is
pinned against torch's fp64 SDPA with ``enable_gqa`` and against the plain multi-head path
on explicitly repeated K/V.  Packed sequences are pinned against the document mask over the
concatenation (a different branch of the oracle) and against separate batch entries."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from attn_workloads import MASK_CAUSAL, MASK_DOC, MASK_NONE, MASK_WINDOW, alibi_slopes, doc_ids_from_lengths
from oracle.attention import attention_fwd, attention_fwd_varlen


def _qkv(B, H, Hkv, Sq, Sk, D, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(B, H, Sq, D, generator=g, dtype=torch.float64),
            torch.randn(B, Hkv, Sk, D, generator=g, dtype=torch.float64),
            torch.randn(B, Hkv, Sk, D, generator=g, dtype=torch.float64))


@pytest.mark.parametrize("H,Hkv", [(8, 1), (8, 2), (8, 4), (6, 3)])
@pytest.mark.parametrize("causal", [False, True])
def test_gqa_library_pin(H, Hkv, causal):
    q, k, v = _qkv(2, H, Hkv, 21, 21, 16, seed=H * 10 + Hkv)
    O, _ = attention_fwd(q, k, v, 0.25, MASK_CAUSAL if causal else MASK_NONE)
    ref = F.scaled_dot_product_attention(q, k, v, is_causal=causal, scale=0.25, enable_gqa=True)
    np.testing.assert_allclose(O, ref.numpy(), rtol=0, atol=1e-12)


def test_gqa_equals_repeated_heads():
    q, k, v = _qkv(1, 8, 2, 30, 40, 8, seed=4)
    sl = alibi_slopes(8).double().numpy()
    args = (0.3, MASK_CAUSAL | MASK_WINDOW, 9, 2.5, sl)
    O1, L1 = attention_fwd(q, k, v, *args)
    O2, L2 = attention_fwd(q, k.repeat_interleave(4, 1), v.repeat_interleave(4, 1), *args)
    np.testing.assert_array_equal(O1, O2)
    np.testing.assert_array_equal(L1, L2)


def test_gqa_rejects_non_dividing_heads():
    q, k, v = _qkv(1, 6, 4, 8, 8, 8, seed=0)
    with pytest.raises(ValueError):
        attention_fwd(q, k, v, 0.3)


def _pack(x):  # [1, H, T, D] -> [T, H, D]
    return x[0].permute(1, 0, 2).contiguous()


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_equals_document_mask(causal):
    """Equal query and key lengths: packed sequences are the document mask over the
    concatenation (bottom-right causal = top-left causal per sequence)."""
    lens = [1, 127, 128, 129, 40, 300]
    T = sum(lens)
    q, k, v = _qkv(1, 4, 2, T, T, 16, seed=8)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    mask = MASK_CAUSAL if causal else MASK_NONE
    O, L = attention_fwd_varlen(_pack(q), _pack(k), _pack(v), cu, cu, 0.25, mask)
    doc = doc_ids_from_lengths(lens)[None]
    Od, Ld = attention_fwd(q, k, v, 0.25, mask | MASK_DOC, 0, 0.0, None, doc)
    np.testing.assert_allclose(O, _pack(torch.from_numpy(Od)).numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(L, Ld[0], rtol=0, atol=1e-12)


def test_varlen_unequal_lengths_match_separate_batches():
    """Sequences with Sq != Sk (bottom-right causal, window, ALiBi positions per sequence)
    equal separate single-sequence calls; an empty query sequence is allowed."""
    lq, lk = [5, 0, 33, 17], [9, 4, 20, 17]
    cq = np.concatenate([[0], np.cumsum(lq)]).astype(np.int32)
    ck = np.concatenate([[0], np.cumsum(lk)]).astype(np.int32)
    H, Hkv, D = 4, 2, 8
    g = torch.Generator().manual_seed(2)
    q = torch.randn(sum(lq), H, D, generator=g, dtype=torch.float64)
    k = torch.randn(sum(lk), Hkv, D, generator=g, dtype=torch.float64)
    v = torch.randn(sum(lk), Hkv, D, generator=g, dtype=torch.float64)
    sl = alibi_slopes(H).double().numpy()
    args = (0.4, MASK_CAUSAL | MASK_WINDOW, 6, 0.0, sl)
    O, L = attention_fwd_varlen(q, k, v, cq, ck, *args)
    for s in range(4):
        if lq[s] == 0:
            continue
        qs = q[cq[s]:cq[s + 1]].permute(1, 0, 2)[None]
        ks = k[ck[s]:ck[s + 1]].permute(1, 0, 2)[None]
        vs = v[ck[s]:ck[s + 1]].permute(1, 0, 2)[None]
        o, l = attention_fwd(qs, ks, vs, *args)
        # each sequence equals a call on that sequence alone
        np.testing.assert_allclose(O[cq[s]:cq[s + 1]], o[0].transpose(1, 0, 2), rtol=0, atol=0)
        np.testing.assert_allclose(L[:, cq[s]:cq[s + 1]], l[0], rtol=0, atol=0)
    # the causal part alone against torch (lower-right causal bias, no window, no ALiBi),
    # on the sequence with fewer queries than keys
    from torch.nn.attention.bias import causal_lower_right
    O2, _ = attention_fwd_varlen(q, k, v, cq, ck, 0.4, MASK_CAUSAL)
    s = 0
    qs = q[cq[s]:cq[s + 1]].permute(1, 0, 2)[None]
    ks = k[ck[s]:ck[s + 1]].permute(1, 0, 2)[None].repeat_interleave(2, 1)
    vs = v[ck[s]:ck[s + 1]].permute(1, 0, 2)[None].repeat_interleave(2, 1)
    ref = F.scaled_dot_product_attention(qs, ks, vs, attn_mask=causal_lower_right(lq[s], lk[s]), scale=0.4)
    np.testing.assert_allclose(O2[cq[s]:cq[s + 1]], ref[0].permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)
