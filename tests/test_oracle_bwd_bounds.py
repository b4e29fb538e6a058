"""The backward parity gate (tests/bwd_bounds.py) checked on the CPU before any kernel
uses it: an emulation of the kernels' arithmetic — bf16 inputs, O rounded to bf16 by the
forward, P, P * dt/ds and dS rounded to bf16 as tensor-core operands, bf16 outputs —
stays inside the bound, and plausible mistakes (a dropped Dv, a missing soft-capping
derivative, a transposed operand) fall outside it."""
import math

import numpy as np
import pytest
import torch

from attn_workloads import MASK_CAUSAL, MASK_DOC, MASK_NONE, MASK_WINDOW, alibi_slopes, doc_ids_from_lengths
from oracle.attention import modified_scores, softmax_rows, visible_mask
from tests.bwd_bounds import bwd_bounds


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).double().numpy()


def _emulate(q, k, v, do, scale, mask, window, softcap, slopes, doc, mistake=None):
    """The kernels' arithmetic in fp64 with their bf16 roundings."""
    B, H, Sq, D = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    G = H // Hkv
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    rows = np.arange(Sq)
    for b in range(B):
        vis = visible_mask(rows, Sq, Sk, mask, window, None if doc is None else doc[b])
        for h in range(H):
            hk = h // G
            t = modified_scores(q[b, h], k[b, hk], scale, rows, Sq, Sk, softcap, None if slopes is None else slopes[h])
            P, m, l = softmax_rows(t, vis)
            O = _bf16(P @ v[b, hk])                        # the forward's bf16 output
            Pb = _bf16(P)
            dv[b, hk] += Pb.T @ do[b, h]
            dP = do[b, h] @ v[b, hk].T
            Dv = (do[b, h] * O).sum(axis=1, keepdims=True)
            if mistake == "drop_dv":
                Dv = 0.0 * Dv
            if softcap > 0 and mistake != "drop_softcap":
                th = np.tanh((q[b, h] @ k[b, hk].T) * scale / softcap)
                fp = 1.0 - th * th
            else:
                fp = 1.0
            dS = _bf16(_bf16(P * fp) * (dP - Dv))
            if mistake == "transpose":
                dS = dS.T if dS.shape[0] == dS.shape[1] else dS
            dq[b, h] = scale * (dS @ k[b, hk])
            dk[b, hk] += scale * (dS.T @ q[b, h])
    return _bf16(dq), _bf16(dk), _bf16(dv)


def _inputs(B, H, Hkv, S, D, seed):
    g = torch.Generator().manual_seed(seed)
    mk = lambda h: torch.randn(B, h, S, D, generator=g).to(torch.bfloat16).double().numpy()
    return mk(H), mk(Hkv), mk(Hkv), mk(H)


CASES = [
    dict(mask=MASK_CAUSAL, window=0, softcap=0.0, alibi=False, H=4, Hkv=2),
    dict(mask=MASK_NONE, window=0, softcap=0.0, alibi=True, H=2, Hkv=2),
    dict(mask=MASK_CAUSAL | MASK_WINDOW, window=40, softcap=0.0, alibi=False, H=2, Hkv=1),
    dict(mask=MASK_NONE, window=0, softcap=3.0, alibi=False, H=2, Hkv=2),
    dict(mask=MASK_DOC, window=0, softcap=0.0, alibi=False, H=2, Hkv=2),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"m{c['mask']}w{c['window']}s{c['softcap']}a{c['alibi']}g{c['H'] // c['Hkv']}")
def test_emulated_kernel_arithmetic_within_bound(case):
    S, D, scale = 160, 32, 1.0 / math.sqrt(32)
    q, k, v, do = _inputs(1, case["H"], case["Hkv"], S, D, seed=case["mask"] + case["H"])
    slopes = alibi_slopes(case["H"]).double().numpy() if case["alibi"] else None
    doc = doc_ids_from_lengths([50, 1, 70, 39])[None] if case["mask"] & MASK_DOC else None
    args = (scale, case["mask"], case["window"], case["softcap"], slopes, doc)
    ref, bnd = bwd_bounds(q, k, v, do, *args)
    got = _emulate(q, k, v, do, *args)
    for g, r, bd, name in zip(got, ref, bnd, ("dQ", "dK", "dV")):
        excess = float((np.abs(g - r) - bd).max())
        assert excess <= 0.0, (name, excess)


@pytest.mark.parametrize("mistake,case", [("drop_dv", CASES[0]), ("drop_softcap", CASES[3]), ("transpose", CASES[1])])
def test_plausible_mistakes_fall_outside_the_bound(mistake, case):
    S, D, scale = 160, 32, 1.0 / math.sqrt(32)
    q, k, v, do = _inputs(1, case["H"], case["Hkv"], S, D, seed=7)
    slopes = alibi_slopes(case["H"]).double().numpy() if case["alibi"] else None
    args = (scale, case["mask"], case["window"], case["softcap"], slopes, None)
    ref, bnd = bwd_bounds(q, k, v, do, *args)
    got = _emulate(q, k, v, do, *args, mistake=mistake)
    worst = max(float((np.abs(g - r) - bd).max()) for g, r, bd in zip(got, ref, bnd))
    assert worst > 0.0
