"""Pins for the fp64 backward oracle (CPU only).

The oracle's gradients are the hand-derived chain rule of the forward definition.  They are
checked against things other than themselves: torch's automatic differentiation of its own
fp64 SDPA (an explicit additive bias carries every mask and ALiBi), automatic
differentiation of a plain torch expression with soft-capping, central finite differences
of the forward oracle on tiny inputs, and invariants of the softmax gradient."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from attn_workloads import (MASK_CAUSAL, MASK_DOC, MASK_NONE, MASK_WINDOW, alibi_slopes,
                            doc_ids_from_lengths, make_qkv)
from oracle.attention import attention_fwd, visible_mask
from oracle.attention_bwd import attention_bwd


def _inputs(B, H, Hkv, Sq, Sk, D, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H, Sq, D, generator=g, dtype=torch.float64)
    k = torch.randn(B, Hkv, Sk, D, generator=g, dtype=torch.float64)
    v = torch.randn(B, Hkv, Sk, D, generator=g, dtype=torch.float64)
    do = torch.randn(B, H, Sq, D, generator=g, dtype=torch.float64)
    return q, k, v, do


def _bias(B, H, Sq, Sk, mask, window, slopes, doc):
    """Additive fp64 bias [B, H, Sq, Sk]: -inf where masked, ALiBi elsewhere."""
    bias = np.zeros((B, H, Sq, Sk))
    rows = np.arange(Sq)
    for b in range(B):
        vis = visible_mask(rows, Sq, Sk, mask, window, None if doc is None else doc[b])
        for h in range(H):
            if slopes is not None:
                ip = rows[:, None] + (Sk - Sq)
                bias[b, h] = slopes[h] * (np.arange(Sk)[None, :] - ip)
            bias[b, h] = np.where(vis, bias[b, h], -np.inf)
    return torch.from_numpy(bias)


def _autograd_sdpa(q, k, v, do, scale, bias):
    q, k, v = (t.clone().requires_grad_(True) for t in (q, k, v))
    G = q.shape[1] // k.shape[1]
    kk, vv = k.repeat_interleave(G, dim=1), v.repeat_interleave(G, dim=1)
    o = F.scaled_dot_product_attention(q, kk, vv, attn_mask=bias, scale=scale)
    o = torch.nan_to_num(o)        # rows with nothing visible: the oracle's O = 0
    (o * do).sum().backward()
    return q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


@pytest.mark.parametrize("mask,window,alibi,H,Hkv,Sq,Sk", [
    (MASK_NONE, 0, False, 2, 2, 37, 29),
    (MASK_CAUSAL, 0, False, 4, 2, 40, 40),
    (MASK_CAUSAL, 0, False, 2, 2, 25, 41),          # bottom-right alignment, Sq < Sk
    (MASK_CAUSAL, 0, False, 2, 2, 41, 25),          # first rows see nothing
    (MASK_CAUSAL | MASK_WINDOW, 7, True, 4, 1, 33, 33),
    (MASK_WINDOW, 5, False, 2, 1, 30, 36),
    (MASK_NONE, 0, True, 4, 4, 20, 20),
])
def test_library_pin_autograd_sdpa(mask, window, alibi, H, Hkv, Sq, Sk):
    q, k, v, do = _inputs(2, H, Hkv, Sq, Sk, 16, seed=Sq * 7 + Sk)
    slopes = alibi_slopes(H).double().numpy() if alibi else None
    scale = 0.37
    dq, dk, dv = attention_bwd(q, k, v, do, scale, mask, window, 0.0, slopes)
    rq, rk, rv = _autograd_sdpa(q, k, v, do, scale, _bias(2, H, Sq, Sk, mask, window, slopes, None))
    for a, r in ((dq, rq), (dk, rk), (dv, rv)):
        np.testing.assert_allclose(a, r, rtol=0, atol=1e-10)


def test_library_pin_document_mask():
    lens = [5, 1, 9, 7]
    S = sum(lens)
    doc = np.stack([doc_ids_from_lengths(lens), doc_ids_from_lengths(lens[::-1])])
    q, k, v, do = _inputs(2, 2, 2, S, S, 8, seed=3)
    for mask in (MASK_DOC, MASK_DOC | MASK_CAUSAL):
        dq, dk, dv = attention_bwd(q, k, v, do, 0.5, mask, 0, 0.0, None, doc)
        rq, rk, rv = _autograd_sdpa(q, k, v, do, 0.5, _bias(2, 2, S, S, mask, 0, None, doc))
        for a, r in ((dq, rq), (dk, rk), (dv, rv)):
            np.testing.assert_allclose(a, r, rtol=0, atol=1e-10)


def test_autograd_pin_softcap_with_alibi_causal():
    """Soft-capping is not an SDPA option: autograd of the plain torch expression."""
    H, S, D, c, scale = 2, 23, 8, 1.7, 0.45
    q, k, v, do = _inputs(1, H, H, S, S, D, seed=11)
    slopes = alibi_slopes(H).double()
    qq, kk, vv = (t.clone().requires_grad_(True) for t in (q, k, v))
    s = (qq @ kk.transpose(-1, -2)) * scale
    t = c * torch.tanh(s / c)
    i = torch.arange(S, dtype=torch.float64)
    t = t + slopes[None, :, None, None] * (i[None, :] - i[:, None])[None, None]
    t = t.masked_fill(torch.ones(S, S, dtype=torch.bool).triu(1), float("-inf"))
    o = torch.softmax(t, dim=-1) @ vv
    (o * do).sum().backward()
    dq, dk, dv = attention_bwd(q, k, v, do, scale, MASK_CAUSAL, 0, c, slopes.numpy())
    for a, r in ((dq, qq.grad), (dk, kk.grad), (dv, vv.grad)):
        np.testing.assert_allclose(a, r.numpy(), rtol=0, atol=1e-10)


@pytest.mark.parametrize("mask,window,softcap,alibi,Hkv", [
    (MASK_NONE, 0, 0.0, False, 2), (MASK_CAUSAL, 0, 2.0, True, 1),
    (MASK_CAUSAL | MASK_WINDOW, 3, 0.0, True, 2), (MASK_DOC, 0, 1.5, False, 1)])
def test_finite_differences(mask, window, softcap, alibi, Hkv):
    """Central differences of L = sum(dO * O) through the forward oracle, every input."""
    H, Sq, Sk, D = 2, 7, 7, 4
    q, k, v, do = (t.numpy() for t in _inputs(1, H, Hkv, Sq, Sk, D, seed=5))
    doc = np.array([[0, 0, 0, 1, 1, 2, 2]]) if mask & MASK_DOC else None
    slopes = alibi_slopes(H).double().numpy() if alibi else None
    scale = 0.8
    args = (scale, mask, window, softcap, slopes, doc)

    def loss(qq, kk, vv):
        return float((attention_fwd(qq, kk, vv, *args)[0] * do).sum())

    dq, dk, dv = attention_bwd(q, k, v, do, *args)
    eps = 1e-6
    for x, g, which in ((q, dq, 0), (k, dk, 1), (v, dv, 2)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            a = [q, k, v]
            a[which] = xp
            lp = loss(*a)
            a[which] = xm
            lm = loss(*a)
            num[idx] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(g, num, rtol=0, atol=1e-7)


def test_zero_keys_give_zero_query_gradient_and_closed_form_dv():
    """K = 0: every visible key weighs 1/n_i, so dQ = 0 and dV_j = sum over rows that see
    j of dO_i / n_i."""
    S, D = 19, 8
    q, _, v, do = (t.numpy() for t in _inputs(1, 1, 1, S, S, D, seed=9))
    k = np.zeros_like(v)
    dq, _, dv = attention_bwd(q, k, v, do, 0.3, MASK_CAUSAL)
    np.testing.assert_allclose(dq, 0.0, atol=1e-13)
    ref = np.zeros((S, D))
    for i in range(S):
        ref[: i + 1] += do[0, 0, i] / (i + 1)
    np.testing.assert_allclose(dv[0, 0], ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("mask,window,alibi", [(MASK_NONE, 0, False), (MASK_CAUSAL, 0, True),
                                               (MASK_WINDOW, 4, False)])
def test_key_gradients_sum_to_zero(mask, window, alibi):
    """Adding one vector to every key moves each row's scores by a constant, which the
    softmax ignores (ALiBi and masks do not depend on K): sum_j dK_j = 0."""
    q, k, v, do = _inputs(2, 2, 2, 15, 18, 8, seed=13)
    slopes = alibi_slopes(2).double().numpy() if alibi else None
    _, dk, _ = attention_bwd(q, k, v, do, 0.6, mask, window, 0.0, slopes)
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-11)


def test_rows_without_keys_contribute_nothing():
    """Causal with Sq > Sk: the first Sq - Sk rows see no key; their dQ is 0 and removing
    them leaves dK and dV unchanged."""
    Sq, Sk = 12, 5
    q, k, v, do = _inputs(1, 2, 2, Sq, Sk, 8, seed=17)
    dq, dk, dv = attention_bwd(q, k, v, do, 0.5, MASK_CAUSAL)
    np.testing.assert_allclose(dq[:, :, : Sq - Sk], 0.0, atol=0)
    dq2, dk2, dv2 = attention_bwd(q[:, :, Sq - Sk:], k, v, do[:, :, Sq - Sk:], 0.5, MASK_CAUSAL)
    np.testing.assert_allclose(dk, dk2, atol=1e-12)
    np.testing.assert_allclose(dv, dv2, atol=1e-12)
    np.testing.assert_allclose(dq[:, :, Sq - Sk:], dq2, atol=1e-12)
