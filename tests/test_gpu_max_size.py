"""GPU parity at the longest sequence the C-ABI accepts (Sq = Sk = ATTN_MAX_SEQ = 2^20, one
head, D = 128), against the fp64 oracle (the FP4 forward against the FP4 oracle).

Forward: sampled query rows, each exact given the full K and V (first rows, both sides of
a 256-row block boundary, the middle, the last rows and random ones), with the BF16 gate.

Backward, causal: key j is seen only by the rows i >= j, so the last 64 keys are seen only by
the last 64 rows.  For those rows the full softmax rows, dP and dS fit in memory, which gives
exact fp64 references for dQ of the 64 rows and for dK, dV of the 64 keys (the last key tile's
work item).  Each element is held to the per-element bound of tests/bwd_bounds.py, computed
over the same rows.  The first rows, which see a handful of keys, are checked the same way."""
import math

import numpy as np
import pytest
import torch

from attn_workloads import MASK_CAUSAL, MASK_NONE, make_qkv, sample_rows
from oracle.attention import modified_scores, softmax_rows, visible_mask
from tests.bwd_bounds import ATOL, EPS, REL_OUT
from tests.gpu_helpers import compare, oracle_eav, to_dev
from tiled_attention_14_b200 import _lib

pytestmark = pytest.mark.gpu

S_MAX = 1 << 20     # ATTN_MAX_SEQ of include/attn.h
D = 128


def _inputs(seed):
    q, k, v = make_qkv(1, 1, S_MAX, S_MAX, D, seed=seed)
    return q, k, v


@pytest.mark.parametrize("mask", [MASK_NONE, MASK_CAUSAL])
def test_forward_at_the_maximum_length(mask):
    import tiled_attention_14_b200 as ta
    q, k, v = _inputs(seed=70 + mask)
    qd, kd, vd = to_dev(q, k, v)
    o, lse = ta.attn_fwd(qd, kd, vd, mask_kind=mask)
    torch.cuda.synchronize()
    assert ta.attn_get_status() == _lib.ATTN_OK
    rows = sample_rows(S_MAX, 6, seed=3, extra=[0, 1, 255, 256, S_MAX // 2, S_MAX - 2, S_MAX - 1])
    O, L, E = oracle_eav(q, k, v, 1.0 / math.sqrt(D), mask, rows=rows)
    compare(o, lse, O, L, rows=rows, eav=E)


def _bwd_reference(q, k, v, do, rows, keys, S=S_MAX):
    """fp64 dQ of `rows` and dK, dV of `keys` (every row that sees a key in `keys` must be in
    `rows`), with their per-element bounds; causal mask, no score modification."""
    scale = 1.0 / math.sqrt(D)
    kf = k[0, 0].double().numpy()
    vf = v[0, 0].double().numpy()
    qr = q[0, 0, rows].double().numpy()
    dor = do[0, 0, rows].double().numpy()
    vis = visible_mask(rows, S, S, MASK_CAUSAL, 0, None)
    t = modified_scores(qr, kf, scale, rows, S, S, 0.0, None)
    P, _, _ = softmax_rows(t, vis)
    del t
    O = P @ vf
    dP = dor @ vf.T
    Dv = (P * dP).sum(axis=1, keepdims=True)
    dS = P * (dP - Dv)
    del dP
    A = (np.abs(dor) * np.abs(O)).sum(axis=1, keepdims=True)
    W = np.abs(dS) + P * A
    dQ = scale * (dS @ kf)
    Tq = scale * (W @ np.abs(kf))
    dK = scale * (dS[:, keys].T @ qr)
    Tk = scale * (W[:, keys].T @ np.abs(qr))
    dV = P[:, keys].T @ dor
    Tv = P[:, keys].T @ np.abs(dor)
    bound = lambda T, g: EPS * T + REL_OUT * np.abs(g) + ATOL
    return (dQ, dK, dV), (bound(Tq, dQ), bound(Tk, dK), bound(Tv, dV))


def test_backward_at_the_maximum_length_causal():
    import tiled_attention_14_b200 as ta
    q, k, v = _inputs(seed=72)
    g = torch.Generator().manual_seed(73)
    do = torch.randn(1, 1, S_MAX, D, generator=g).to(torch.bfloat16)
    qd, kd, vd, dod = to_dev(q, k, v, do)
    o, lse = ta.attn_fwd(qd, kd, vd, mask_kind=MASK_CAUSAL)
    dq, dk, dv = ta.attn_bwd(qd, kd, vd, o, lse, dod, mask_kind=MASK_CAUSAL)
    torch.cuda.synchronize()
    assert ta.attn_get_status() == _lib.ATTN_OK
    tail = np.arange(S_MAX - 64, S_MAX)
    for rows, keys in ((tail, tail), (np.arange(0, 4), np.arange(0, 0))):
        ref, bnd = _bwd_reference(q, k, v, do, rows, keys)
        got = (dq[0, 0, rows], dk[0, 0, keys], dv[0, 0, keys])
        for name, gg, r, bd in zip(("dQ", "dK", "dV"), got, ref, bnd):
            if r.size == 0:
                continue
            gv = gg.float().cpu().numpy().astype(np.float64)
            assert np.all(np.isfinite(gv)), name
            excess = float((np.abs(gv - r) - bd).max())
            assert excess <= 0.0, f"{name}: max|err| {np.abs(gv - r).max():.3e} exceeds the bound by {excess:.3e}"


def test_fp4_forward_at_the_maximum_length():
    """The FP4 Direct-P forward at 2^20 queries and keys, sampled rows, against the FP4 oracle
    on its own MXFP4 quantisation of the same inputs."""
    from tests.test_gpu_fp4 import _check
    q, k, v = _inputs(seed=74)
    rows = sample_rows(S_MAX, 4, seed=5, extra=[0, 1, S_MAX // 2, S_MAX - 1])
    _check(q, k, v, rows=rows)
