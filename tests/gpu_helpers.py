"""Shared helpers of the GPU parity tests: run the CUDA path through the C-ABI and compare
it element by element with the fp64 oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

from oracle.attention import attention_fwd

# Tolerances of the BF16 path (bf16 inputs, fp32 accumulation).
TOL_O_BF16 = 1e-2
TOL_LSE_BF16 = 1e-3
# Two roundings are part of the method and no kernel can avoid them: P is rounded to bf16
# before P.V (moving O by at most 2^-8 E_p|v|, E_p|v| the softmax-weighted mean of |v|) and
# O itself is stored in bf16 (half an ulp, at most 2^-8 |O|: bf16 keeps 8 significant bits).  In rows that see few keys
# with large values they alone exceed 1e-2 (tests/test_oracle_bf16_floor.py shows it on a
# test input), so every element is held to 1e-2 + 2^-8 (|O| + E_p|v|).
ROUND_BF16 = 2.0 ** -8
# kept for callers that pass a relative term of their own
TOL_REL_STRESS = 2.0 ** -8
# FP8 path.
TOL_O_FP8 = 5e-2
TOL_COS_FP8 = 0.999


def to_dev(*ts):
    return [None if t is None else t.cuda().contiguous() for t in ts]


def compare(o_gpu, lse_gpu, O_ref, L_ref, tol_o=TOL_O_BF16, tol_lse=TOL_LSE_BF16, rows=None,
            tol_rel=0.0, eav=None):
    """Returns (max|dO|, max|dLSE|) after checking -inf rows agree exactly.  With ``eav``
    (E_p|v| per element, from the oracle run on |V|) each element is held to
    tol_o + 2^-8 (|O| + E_p|v|): the absolute gate plus the bf16 roundings of P and O."""
    o = o_gpu.float().cpu().numpy().astype(np.float64)
    lse = lse_gpu.float().cpu().numpy().astype(np.float64)
    if rows is not None:
        o = o[:, :, rows]
        lse = lse[:, :, rows]
    ninf_ref = np.isneginf(L_ref)
    assert np.array_equal(np.isneginf(lse), ninf_ref), "rows with no visible key differ"
    assert np.all(o[ninf_ref] == 0.0)
    assert np.all(np.isfinite(o)), "non-finite output"
    fin = ~ninf_ref
    err = np.abs(o - O_ref)
    dO = float(err.max()) if o.size else 0.0
    dL = float(np.abs(lse[fin] - L_ref[fin]).max()) if fin.any() else 0.0
    if eav is not None:
        bound = tol_o + tol_rel * np.abs(O_ref) + ROUND_BF16 * (np.abs(O_ref) + eav)
        excess = float((err - bound).max()) if o.size else 0.0
        assert excess <= 0.0, f"max|dO| = {dO:.3e}; the bound is exceeded by {excess:.3e}"
    elif tol_rel == 0.0:
        assert dO <= tol_o, f"max|dO| = {dO:.3e} > {tol_o}"
    else:
        excess = float((err - (tol_o + tol_rel * np.abs(O_ref))).max()) if o.size else 0.0
        assert excess <= 0.0, f"max|dO| = {dO:.3e} exceeds {tol_o} + {tol_rel:.2e}|O| by {excess:.3e}"
    assert dL <= tol_lse, f"max|dLSE| = {dL:.3e} > {tol_lse}"
    return dO, dL


def oracle(q, k, v, scale, mask_kind=0, window=0, softcap=0.0, alibi=None, doc=None, rows=None):
    return attention_fwd(q, k, v, scale, mask_kind, window, softcap,
                         None if alibi is None else alibi.numpy(), doc, rows=rows)


def oracle_eav(q, k, v, scale, mask_kind=0, window=0, softcap=0.0, alibi=None, doc=None, rows=None):
    """(O, LSE, E_p|v|): the oracle, and the same softmax applied to |V|."""
    O, L = oracle(q, k, v, scale, mask_kind, window, softcap, alibi, doc, rows)
    vabs = v.abs() if hasattr(v, "abs") else np.abs(v)
    E, _ = oracle(q, k, vabs, scale, mask_kind, window, softcap, alibi, doc, rows)
    return O, L, E
