"""GPU parity of the attention backward (attn_bwd, through the C-ABI) against the fp64
oracle's gradients.  The forward kernel supplies O and LSE, as a training step would; each
gradient element is held to the bound of tests/bwd_bounds.py (bf16 operand and output
rounding; checked on the CPU against an emulation of the kernels' arithmetic and against
planted mistakes).  Also: bitwise run-to-run determinism with the tile ranges and the
document mask, rows and key tiles that see nothing, and a head of the causal benchmark
shape at full size."""
import math

import numpy as np
import pytest
import torch

from attn_workloads import (MASK_CAUSAL, MASK_DOC, MASK_NONE, MASK_WINDOW, alibi_slopes, doc_ids_from_lengths,
                            make_qkv)
from tests.bwd_bounds import bwd_bounds
from tests.gpu_helpers import to_dev

pytestmark = pytest.mark.gpu


def _dout(B, H, Sq, D, seed):
    g = torch.Generator().manual_seed(seed + 1000)
    return torch.randn(B, H, Sq, D, generator=g).to(torch.bfloat16)


def _run(B, H, Hkv, Sq, Sk, D, mask=MASK_NONE, window=0, softcap=0.0, alibi=False, doc=None, seed=0):
    import tiled_attention_14_b200 as ta
    q, k, v = make_qkv(B, H, Sq, Sk, D, seed=seed, Hkv=Hkv)
    do = _dout(B, H, Sq, D, seed)
    sl = alibi_slopes(H) if alibi else None
    qd, kd, vd, dod, sld, docd = to_dev(q, k, v, do, sl, doc)
    scale = 1.0 / math.sqrt(D)
    kw = dict(scale=scale, mask_kind=mask, window=window, softcap=softcap, alibi_slopes=sld, doc_ids=docd)
    o, lse = ta.attn_fwd(qd, kd, vd, **kw)
    dq, dk, dv = ta.attn_bwd(qd, kd, vd, o, lse, dod, **kw)
    torch.cuda.synchronize()
    assert ta.attn_get_status() == 0
    ref, bnd = bwd_bounds(q, k, v, do, scale, mask, window, softcap, None if sl is None else sl.numpy(), doc)
    for name, g, r, bd in zip(("dQ", "dK", "dV"), (dq, dk, dv), ref, bnd):
        gg = g.float().cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(gg)), name
        excess = float((np.abs(gg - r) - bd).max())
        assert excess <= 0.0, f"{name}: max|err| = {np.abs(gg - r).max():.3e}, exceeds the bound by {excess:.3e}"
    return dq, dk, dv


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("Sq,Sk", [(128, 128), (300, 300), (520, 200), (200, 520), (1, 129)])
@pytest.mark.parametrize("mask", [MASK_NONE, MASK_CAUSAL])
def test_shapes(D, Sq, Sk, mask):
    _run(1, 2, 2, Sq, Sk, D, mask, seed=Sq * 3 + Sk + mask)


@pytest.mark.parametrize("H,Hkv", [(4, 2), (4, 1)])
def test_grouped_heads(H, Hkv):
    _run(2, H, Hkv, 400, 400, 128, MASK_CAUSAL, seed=H + Hkv)


@pytest.mark.parametrize("mask,window", [(MASK_CAUSAL | MASK_WINDOW, 100), (MASK_WINDOW, 70), (MASK_WINDOW, 1)])
def test_window(mask, window):
    _run(1, 2, 2, 500, 500, 128, mask, window=window, seed=window)


def test_alibi_and_softcap():
    _run(1, 4, 4, 330, 330, 128, MASK_CAUSAL, alibi=True, seed=1)
    _run(1, 2, 2, 300, 300, 128, MASK_NONE, softcap=5.0, seed=2)
    _run(1, 2, 1, 260, 260, 64, MASK_CAUSAL, softcap=20.0, alibi=True, seed=3)


@pytest.mark.parametrize("causal", [False, True])
def test_document_mask(causal):
    lens = [300, 129, 1, 450, 144]
    S = sum(lens)
    doc = torch.from_numpy(np.stack([doc_ids_from_lengths(lens), doc_ids_from_lengths(lens[::-1])]))
    _run(2, 2, 2, S, S, 128, MASK_DOC | (MASK_CAUSAL if causal else 0), doc=doc, seed=S)


def test_document_mask_unsorted_ids():
    rng = np.random.default_rng(4)
    doc = torch.from_numpy(rng.integers(0, 3, size=(1, 390)).astype(np.int32))
    _run(1, 2, 2, 390, 390, 128, MASK_DOC, doc=doc, seed=5)


def test_deterministic():
    import tiled_attention_14_b200 as ta
    lens = [700, 324]
    doc = torch.from_numpy(doc_ids_from_lengths(lens)[None].repeat(2, 0)).cuda()
    q, k, v = to_dev(*make_qkv(2, 4, 1024, 1024, 128, seed=6, Hkv=2))
    do = _dout(2, 4, 1024, 128, 6).cuda()
    for mask in (MASK_CAUSAL, MASK_DOC | MASK_CAUSAL):
        o, lse = ta.attn_fwd(q, k, v, mask_kind=mask, doc_ids=doc)
        a = ta.attn_bwd(q, k, v, o, lse, do, mask_kind=mask, doc_ids=doc)
        b = ta.attn_bwd(q, k, v, o, lse, do, mask_kind=mask, doc_ids=doc)
        torch.cuda.synchronize()
        for x, y in zip(a, b):
            assert torch.equal(x, y)


def test_full_size_causal_one_head():
    """The causal benchmark shape (B4 H16 S4096 D128); the oracle checks heads (0, 0) and
    (3, 15) in full."""
    import tiled_attention_14_b200 as ta
    B, H, S, D = 4, 16, 4096, 128
    q, k, v = make_qkv(B, H, S, S, D, seed=0)
    do = _dout(B, H, S, D, 0)
    qd, kd, vd, dod = to_dev(q, k, v, do)
    o, lse = ta.attn_fwd(qd, kd, vd, mask_kind=MASK_CAUSAL)
    dq, dk, dv = ta.attn_bwd(qd, kd, vd, o, lse, dod, mask_kind=MASK_CAUSAL)
    torch.cuda.synchronize()
    assert ta.attn_get_status() == 0
    for b, h in ((0, 0), (3, 15)):
        sl = lambda t: t[b:b + 1, h:h + 1]
        ref, bnd = bwd_bounds(sl(q), sl(k), sl(v), sl(do), 1.0 / math.sqrt(D), MASK_CAUSAL)
        for name, g, r, bd in zip(("dQ", "dK", "dV"), (dq, dk, dv), ref, bnd):
            gg = sl(g).float().cpu().numpy().astype(np.float64)
            excess = float((np.abs(gg - r) - bd).max())
            assert excess <= 0.0, (name, b, h, excess)
