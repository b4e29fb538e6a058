"""GPU parity of the FP4 path against the oracle, through the C-ABI.

The MXFP4 quantiser is compared bit for bit (codes and E8M0 scale atoms, in the layout
include/attn.h states) with the oracle quantiser.  The Direct-P forward is compared element
by element with the fp64 oracle run on the oracle's own dequantised inputs, within the bound
of tests/fp4_bounds.py (neighbouring codes where a score sits on a code boundary within the
fp32 accumulation error, plus the bf16 rounding of O)."""
import math

import numpy as np
import pytest
import torch

from attn_workloads import make_qkv, sample_rows
from tests.fp4_bounds import dequantised, expected_rows, expected_transposed, reference_with_bound
from tiled_attention_14_b200 import _lib

pytestmark = pytest.mark.gpu

TOL_ABS_O = 1e-3
TOL_REL_O = 2.0 ** -8      # bf16 output rounding (half an ulp is 2^-9 of |O|)
TOL_LSE = 1e-4


def _quantise_all(q, k, v):
    import tiled_attention_14_b200 as ta
    qd, kd, vd = (x.cuda().contiguous() for x in (q, k, v))
    q4, qsf = ta.attn_quantize_mxfp4(qd)
    k4, ksf = ta.attn_quantize_mxfp4(kd)
    v4, vsf = ta.attn_quantize_mxfp4(vd, transpose=True)
    return q4, qsf, k4, ksf, v4, vsf


def _check(q, k, v, rows=None, scale=None, heads=None):
    """Runs the FP4 path on the whole problem and compares the query rows `rows` of the
    query heads `heads` (all if None; grouped heads need all)."""
    import tiled_attention_14_b200 as ta
    B, H, Sq, D = q.shape
    Sk = k.shape[2]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    q4, qsf, k4, ksf, v4, vsf = _quantise_all(q, k, v)
    o, lse = ta.attn_fwd_fp4(q4, qsf, k4, ksf, v4, vsf, Sk, scale=scale)
    torch.cuda.synchronize()
    assert ta.attn_get_status() == _lib.ATTN_OK
    rows = np.arange(Sq) if rows is None else np.asarray(rows)
    hs = slice(None) if heads is None else list(heads)
    qn, kn, vn = (x[:, hs].float().numpy() for x in (q, k, v))
    qh, kh, vh = dequantised(qn, kn, vn)
    O, L, bO, bL = reference_with_bound(qh, kh, vh, scale, rows)
    og = o[:, hs].float().cpu().numpy()[:, :, rows].astype(np.float64)
    lg = lse[:, hs].float().cpu().numpy()[:, :, rows].astype(np.float64)
    assert np.all(np.isfinite(og)) and np.all(np.isfinite(lg))
    err = np.abs(og - O)
    lim = TOL_ABS_O + TOL_REL_O * np.abs(O) + 1.05 * bO
    excess = err - lim
    i = np.unravel_index(np.argmax(excess), excess.shape)
    assert excess.max() <= 0.0, (f"O: max excess {excess.max():.3e} at {i}: gpu {og[i]:.6f} oracle {O[i]:.6f} "
                                 f"bound {lim[i]:.3e}; max|dO| {err.max():.3e}")
    lerr = np.abs(lg - L) - (TOL_LSE + 1.05 * bL)
    assert lerr.max() <= 0.0, f"LSE: max excess {lerr.max():.3e}, max|dLSE| {np.abs(lg - L).max():.3e}"
    return err.max(), float(np.abs(lg - L).max())


@pytest.mark.parametrize("B,H,S", [(1, 2, 256), (2, 3, 200), (1, 1, 1), (1, 2, 129), (1, 1, 1000)])
def test_quantiser_rows_bit_exact(B, H, S):
    import tiled_attention_14_b200 as ta
    g = torch.Generator().manual_seed(S)
    x = (torch.randn(B, H, S, 128, generator=g) * torch.exp2(torch.randint(-8, 8, (B, H, S, 1), generator=g))).to(torch.bfloat16)
    x[0, 0, 0, 32:64] = 0.0                      # a zero block
    x[0, -1, -1, :8] = 1e30                      # a large block
    xq, xsf = ta.attn_quantize_mxfp4(x.cuda())
    torch.cuda.synchronize()
    eq, esf = expected_rows(x.float().numpy())
    assert np.array_equal(xq.cpu().numpy(), eq)
    assert np.array_equal(xsf.cpu().numpy(), esf)


@pytest.mark.parametrize("B,H,S", [(1, 2, 256), (2, 1, 300), (1, 1, 1), (1, 1, 64)])
def test_quantiser_transposed_bit_exact(B, H, S):
    import tiled_attention_14_b200 as ta
    g = torch.Generator().manual_seed(7 + S)
    x = torch.randn(B, H, S, 128, generator=g).to(torch.bfloat16)
    x[0, 0, :32, 5] = 0.0                         # a zero block of column 5
    xq, xsf = ta.attn_quantize_mxfp4(x.cuda(), transpose=True)
    torch.cuda.synchronize()
    eq, esf = expected_transposed(x.float().numpy())
    assert np.array_equal(xq.cpu().numpy(), eq)
    assert np.array_equal(xsf.cpu().numpy(), esf)


@pytest.mark.parametrize("B,H,Sq,Sk", [(1, 2, 256, 256), (1, 1, 200, 333), (2, 3, 129, 64), (1, 1, 1, 1),
                                       (1, 2, 512, 1000), (1, 1, 300, 65), (1, 1, 64, 4096)])
def test_fp4_forward_parity(B, H, Sq, Sk):
    q, k, v = make_qkv(B, H, Sq, Sk, 128, seed=B * 1000 + Sq + Sk)
    _check(q, k, v)


def test_fp4_forward_grouped_heads():
    q, k, v = make_qkv(1, 4, 256, 384, 128, seed=11, Hkv=2)
    _check(q, k, v)


def test_fp4_forward_multi_query_unequal_lengths():
    """One K/V head for four query heads, more keys than queries (no mask: every key visible)."""
    q, k, v = make_qkv(2, 4, 300, 700, 128, seed=14, Hkv=1)
    _check(q, k, v)


@pytest.mark.parametrize("mul", [4.0, 0.05])
def test_fp4_forward_peaked_and_flat_rows(mul):
    """Q x 4 moves the row maximum by many octaves across key tiles (the rescale path);
    Q x 0.05 makes every row nearly flat (all codes near the top of their blocks)."""
    q, k, v = make_qkv(1, 2, 256, 1024, 128, seed=12, q_mul=mul)
    _check(q, k, v)


@pytest.mark.parametrize("scale", [0.02, 0.3])
def test_fp4_forward_other_scales(scale):
    """A softmax scale other than 1/sqrt(D): the kernel's score-to-code constant and the
    oracle's both follow the scale argument (small: nearly flat rows; large: peaked rows)."""
    q, k, v = make_qkv(1, 2, 300, 520, 128, seed=15)
    _check(q, k, v, scale=scale)


def test_fp4_forward_full_size_sampled_rows():
    """The non-causal inference shape (B1 H32 S32768 D128), sampled rows of three heads."""
    q, k, v = make_qkv(1, 32, 32768, 32768, 128, seed=0)
    rows = sample_rows(32768, 4, seed=1)
    _check(q, k, v, rows=rows, heads=[0, 13, 31])


def test_fp4_forward_deterministic():
    import tiled_attention_14_b200 as ta
    q, k, v = make_qkv(1, 4, 640, 900, 128, seed=13)
    q4, qsf, k4, ksf, v4, vsf = _quantise_all(q, k, v)
    o1, l1 = ta.attn_fwd_fp4(q4, qsf, k4, ksf, v4, vsf, 900)
    o2, l2 = ta.attn_fwd_fp4(q4, qsf, k4, ksf, v4, vsf, 900)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
