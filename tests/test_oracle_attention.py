"""Pins for the fp64 attention oracle (CPU only).

Each test checks the oracle against something other than itself: hand-derived worked
examples, closed forms, invariants, pure-Python brute force on tiny inputs, or torch's
CPU fp64 SDPA library routine.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle.attention import attention_fwd, visible_mask, visible_pair_count
from attn_workloads import (MASK_CAUSAL, MASK_DOC, MASK_NONE, MASK_WINDOW, alibi_slopes,
                            doc_ids_from_lengths, doc_lengths, make_qkv)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


def _t(a):
    return torch.tensor(a, dtype=torch.float64)


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_worked_examples(case):
    q = np.array(case["q"], dtype=np.float64)[None, None]
    if "k_log_args" in case:
        k = np.log(np.array(case["k_log_args"], dtype=np.float64))[:, None][None, None]
    else:
        k = np.array(case["k"], dtype=np.float64)[None, None]
    v = np.array(case["v"], dtype=np.float64)[None, None]
    doc = None if "doc_ids" not in case else np.array([case["doc_ids"]], dtype=np.int32)
    slopes = case.get("alibi_slopes")
    O, L = attention_fwd(q, k, v, case["scale"], case["mask_kind"], case["window"],
                         case["softcap"], slopes, doc)
    np.testing.assert_allclose(O[0, 0], np.array(case["O"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(L[0, 0], np.array(case["LSE"]), rtol=0, atol=1e-12)


def _rand(B, H, Sq, Sk, D, seed=0):
    q, k, v = make_qkv(B, H, Sq, Sk, D, seed=seed, dtype=torch.float64)
    return q.numpy(), k.numpy(), v.numpy()


@pytest.mark.parametrize("mask,window", [(MASK_NONE, 0), (MASK_CAUSAL, 0),
                                         (MASK_CAUSAL | MASK_WINDOW, 5), (MASK_WINDOW, 3)])
def test_rows_sum_to_one(mask, window):
    """V == 1 makes every visible row's output the sum of its softmax weights."""
    q, k, _ = _rand(1, 2, 17, 23, 8)
    v = np.ones_like(k)
    O, L = attention_fwd(q, k, v, 0.3, mask, window)
    vis = visible_mask(np.arange(17), 17, 23, mask, window, None).any(1)
    np.testing.assert_allclose(O[0, :, vis, :], 1.0, atol=1e-12)


def _mean_visible_closed_form(Sq, Sk, mask, W, i):
    ip = i + Sk - Sq
    if mask == MASK_NONE:
        return 0, Sk - 1
    if mask == MASK_CAUSAL:
        return 0, min(ip, Sk - 1)
    if mask == MASK_CAUSAL | MASK_WINDOW:
        return max(0, ip - W + 1), min(ip, Sk - 1)
    if mask == MASK_WINDOW:
        return max(0, ip - W + 1), min(Sk - 1, ip + W - 1)
    raise AssertionError


@pytest.mark.parametrize("Sq,Sk", [(19, 19), (7, 19), (19, 30)])
@pytest.mark.parametrize("mask,W", [(MASK_NONE, 0), (MASK_CAUSAL, 0),
                                    (MASK_CAUSAL | MASK_WINDOW, 4), (MASK_WINDOW, 4)])
def test_zero_keys_give_mean_of_visible_values(Sq, Sk, mask, W):
    """K == 0: all scores are 0, so O_i is the mean of the visible V rows and
    LSE_i = ln(n_visible), with the visible range in closed form."""
    q, _, v = _rand(1, 1, Sq, Sk, 4, seed=3)
    k = np.zeros((1, 1, Sk, 4))
    O, L = attention_fwd(q, k, v, 1.0, mask, W)
    for i in range(Sq):
        lo, hi = _mean_visible_closed_form(Sq, Sk, mask, W, i)
        if hi < lo:
            assert np.all(O[0, 0, i] == 0) and L[0, 0, i] == -np.inf
            continue
        np.testing.assert_allclose(O[0, 0, i], v[0, 0, lo:hi + 1].mean(0), atol=1e-12)
        assert abs(L[0, 0, i] - math.log(hi - lo + 1)) < 1e-12


def test_zero_keys_document_mask():
    lens = [3, 5, 1, 7]
    doc = doc_ids_from_lengths(lens)[None]
    S = sum(lens)
    q, _, v = _rand(1, 2, S, S, 4, seed=5)
    k = np.zeros_like(q)
    O, L = attention_fwd(q, k, v, 1.0, MASK_DOC, 0, doc_ids=doc)
    start = 0
    for n in lens:
        for i in range(start, start + n):
            np.testing.assert_allclose(O[0, :, i], v[0, :, start:start + n].mean(1), atol=1e-12)
            np.testing.assert_allclose(L[0, :, i], math.log(n), atol=1e-12)
        start += n


def test_alibi_causal_zero_keys_closed_form():
    """K == 0, causal, ALiBi slope m: weights on key i-d are r^d with r = e^-m, so
    LSE_i = ln((1 - r^(i+1)) / (1 - r)) and, with V_j = j,
    O_i = i - sum_d d r^d / sum_d r^d  (arithmetico-geometric series)."""
    S, H = 40, 3
    slopes = np.array([0.5, 0.05, 1.7])
    q = np.random.default_rng(0).standard_normal((1, H, S, 2))
    k = np.zeros((1, H, S, 2))
    v = np.tile(np.arange(S, dtype=np.float64)[:, None], (1, H, 1, 2)).reshape(1, H, S, 2)
    O, L = attention_fwd(q, k, v, 1.0, MASK_CAUSAL, 0, alibi_slopes=slopes)
    for h, m in enumerate(slopes):
        r = math.exp(-m)
        for i in range(S):
            n = i
            geo = (1 - r ** (n + 1)) / (1 - r)
            ag = r * (1 - (n + 1) * r ** n + n * r ** (n + 1)) / (1 - r) ** 2
            assert abs(L[0, h, i] - math.log(geo)) < 1e-12
            assert abs(O[0, h, i, 0] - (i - ag / geo)) < 1e-9


def test_causal_row0_is_v0():
    q, k, v = _rand(2, 3, 9, 9, 16, seed=7)
    O, L = attention_fwd(q, k, v, 0.25, MASK_CAUSAL)
    np.testing.assert_array_equal(O[:, :, 0], v[:, :, 0])
    s00 = 0.25 * np.einsum("bhd,bhd->bh", q[:, :, 0], k[:, :, 0])
    np.testing.assert_allclose(L[:, :, 0], s00, atol=1e-13)


@pytest.mark.parametrize("mask", [MASK_CAUSAL | MASK_WINDOW, MASK_WINDOW])
def test_single_visible_key_returns_that_value(mask):
    q, k, v = _rand(1, 2, 11, 11, 8, seed=2)
    O, L = attention_fwd(q, k, v, 0.5, mask, 1)
    np.testing.assert_array_equal(O[0], v[0])
    diag = 0.5 * np.einsum("hsd,hsd->hs", q[0], k[0])
    np.testing.assert_allclose(L[0], diag, atol=1e-13)


def _brute(q, k, v, scale, mask, W, softcap, slope, doc):
    """Pure-Python double loop over (i, j): scores, mask, log-sum-exp by math.exp."""
    Sq, D = len(q), len(q[0])
    Sk = len(k)
    out, lse = [], []
    for i in range(Sq):
        ip = i + Sk - Sq
        vals = []
        for j in range(Sk):
            ok = True
            if mask & 1 and j > ip:
                ok = False
            if mask & 2:
                if mask & 1 and not (ip - j < W):
                    ok = False
                if not mask & 1 and not (abs(ip - j) < W):
                    ok = False
            if mask & 4 and doc[i] != doc[j]:
                ok = False
            if not ok:
                continue
            s = scale * sum(q[i][d] * k[j][d] for d in range(D))
            if softcap > 0:
                s = softcap * math.tanh(s / softcap)
            if slope is not None:
                s += slope * (j - ip)
            vals.append((j, s))
        if not vals:
            out.append([0.0] * len(v[0]))
            lse.append(-math.inf)
            continue
        mx = max(s for _, s in vals)
        tot = sum(math.exp(s - mx) for _, s in vals)
        lse.append(mx + math.log(tot))
        o = [0.0] * len(v[0])
        for j, s in vals:
            w = math.exp(s - mx) / tot
            for d in range(len(v[0])):
                o[d] += w * v[j][d]
        out.append(o)
    return out, lse


@pytest.mark.parametrize("Sq,Sk", [(6, 6), (4, 8), (8, 5)])
@pytest.mark.parametrize("mask,W,softcap,alibi", [
    (MASK_NONE, 0, 0.0, False), (MASK_CAUSAL, 0, 0.0, False), (MASK_CAUSAL | MASK_WINDOW, 2, 0.0, False),
    (MASK_WINDOW, 2, 0.0, False), (MASK_NONE, 0, 1.5, False), (MASK_CAUSAL, 0, 0.0, True),
    (MASK_CAUSAL, 0, 2.0, True)])
def test_brute_force_tiny(Sq, Sk, mask, W, softcap, alibi):
    q, k, v = _rand(1, 2, Sq, Sk, 3, seed=11)
    slopes = np.array([0.7, 0.2]) if alibi else None
    O, L = attention_fwd(q, k, v, 0.9, mask, W, softcap, slopes)
    for h in range(2):
        bo, bl = _brute(q[0, h].tolist(), k[0, h].tolist(), v[0, h].tolist(), 0.9, mask, W,
                        softcap, None if slopes is None else slopes[h], None)
        np.testing.assert_allclose(O[0, h], np.array(bo), atol=1e-12)
        np.testing.assert_allclose(L[0, h], np.array(bl), atol=1e-12)


def test_brute_force_tiny_document():
    doc = np.array([[0, 0, 0, 1, 2, 2, 2, 2]], dtype=np.int32)
    q, k, v = _rand(1, 1, 8, 8, 3, seed=12)
    for mask in (MASK_DOC, MASK_DOC | MASK_CAUSAL):
        O, L = attention_fwd(q, k, v, 0.8, mask, 0, doc_ids=doc)
        bo, bl = _brute(q[0, 0].tolist(), k[0, 0].tolist(), v[0, 0].tolist(), 0.8, mask, 0, 0.0,
                        None, doc[0].tolist())
        np.testing.assert_allclose(O[0, 0], np.array(bo), atol=1e-12)
        np.testing.assert_allclose(L[0, 0], np.array(bl), atol=1e-12)


def test_lse_bounds():
    q, k, v = _rand(1, 2, 33, 47, 16, seed=4)
    O, L = attention_fwd(q, k, v, 0.5, MASK_NONE)
    s = 0.5 * np.einsum("hid,hjd->hij", q[0], k[0])
    mx = s.max(-1)
    assert np.all(L[0] >= mx - 1e-12)
    assert np.all(L[0] <= mx + math.log(47) + 1e-12)


def test_key_permutation_invariance():
    q, k, v = _rand(1, 2, 21, 29, 8, seed=9)
    perm = np.random.default_rng(1).permutation(29)
    for softcap in (0.0, 3.0):
        O1, L1 = attention_fwd(q, k, v, 0.4, MASK_NONE, softcap=softcap)
        O2, L2 = attention_fwd(q, k[:, :, perm], v[:, :, perm], 0.4, MASK_NONE, softcap=softcap)
        np.testing.assert_allclose(O1, O2, atol=1e-12)
        np.testing.assert_allclose(L1, L2, atol=1e-12)


def test_softcap_large_cap_and_zero_slope_reduce_to_plain():
    q, k, v = _rand(1, 2, 15, 15, 8, seed=6)
    O0, L0 = attention_fwd(q, k, v, 0.3, MASK_CAUSAL)
    O1, L1 = attention_fwd(q, k, v, 0.3, MASK_CAUSAL, softcap=1e9)
    O2, L2 = attention_fwd(q, k, v, 0.3, MASK_CAUSAL, alibi_slopes=np.zeros(2))
    np.testing.assert_allclose(O1, O0, atol=1e-9)
    np.testing.assert_allclose(L1, L0, atol=1e-9)
    np.testing.assert_array_equal(O2, O0)
    np.testing.assert_array_equal(L2, L0)


def _sdpa(q, k, v, scale, bias):
    return torch.nn.functional.scaled_dot_product_attention(_t(q), _t(k), _t(v),
                                                            attn_mask=bias, scale=scale)


@pytest.mark.parametrize("Sq,Sk", [(32, 32), (20, 45)])
def test_library_pin_plain_and_lower_right_causal(Sq, Sk):
    """torch's CPU fp64 SDPA; bottom-right causal from torch's own causal_lower_right."""
    from torch.nn.attention.bias import causal_lower_right
    q, k, v = _rand(2, 3, Sq, Sk, 16, seed=8)
    O, _ = attention_fwd(q, k, v, 0.25, MASK_NONE)
    np.testing.assert_allclose(O, _sdpa(q, k, v, 0.25, None).numpy(), atol=1e-12)
    O, _ = attention_fwd(q, k, v, 0.25, MASK_CAUSAL)
    ref = torch.nn.functional.scaled_dot_product_attention(
        _t(q), _t(k), _t(v), attn_mask=causal_lower_right(Sq, Sk), scale=0.25)
    ref = torch.nan_to_num(ref, nan=0.0).numpy()   # rows with nothing visible
    np.testing.assert_allclose(O, ref, atol=1e-12)


def test_library_pin_sliding_window_alibi_document():
    S, H = 40, 4
    q, k, v = _rand(2, H, S, S, 8, seed=10)
    i = torch.arange(S)[:, None]
    j = torch.arange(S)[None, :]
    # sliding window 6 with causal, as a boolean mask handed to the library
    keep = (j <= i) & (i - j < 6)
    O, _ = attention_fwd(q, k, v, 0.5, MASK_CAUSAL | MASK_WINDOW, 6)
    np.testing.assert_allclose(O, _sdpa(q, k, v, 0.5, keep).numpy(), atol=1e-12)
    # ALiBi with causal as an additive float bias
    sl = alibi_slopes(H).double()
    bias = sl[:, None, None] * (j - i).double()[None]
    bias = bias.masked_fill(~(j <= i)[None], float("-inf"))
    O, _ = attention_fwd(q, k, v, 0.5, MASK_CAUSAL, alibi_slopes=sl.numpy())
    np.testing.assert_allclose(O, _sdpa(q, k, v, 0.5, bias[None]).numpy(), atol=1e-12)
    # document mask, block diagonal
    doc = np.stack([doc_ids_from_lengths([10, 25, 5]), doc_ids_from_lengths([40])])
    O, _ = attention_fwd(q, k, v, 0.5, MASK_DOC, doc_ids=doc)
    dt = torch.from_numpy(doc)
    keep = (dt[:, :, None] == dt[:, None, :])[:, None]
    np.testing.assert_allclose(O, _sdpa(q, k, v, 0.5, keep).numpy(), atol=1e-12)


def test_row_subset_matches_full():
    q, k, v = _rand(1, 2, 50, 50, 8, seed=13)
    O, L = attention_fwd(q, k, v, 0.3, MASK_CAUSAL)
    rows = np.array([0, 7, 49])
    Os, Ls = attention_fwd(q, k, v, 0.3, MASK_CAUSAL, rows=rows)
    np.testing.assert_array_equal(Os, O[:, :, rows])
    np.testing.assert_array_equal(Ls, L[:, :, rows])


def test_visible_pair_count_closed_forms():
    S = 300
    assert visible_pair_count(S, S, MASK_NONE, 0) == S * S
    assert visible_pair_count(S, S, MASK_CAUSAL, 0) == S * (S + 1) // 2
    W = 37
    assert visible_pair_count(S, S, MASK_CAUSAL | MASK_WINDOW, W) == W * (W + 1) // 2 + (S - W) * W
    lens = doc_lengths(8192, 0)
    assert visible_pair_count(8192, 8192, MASK_DOC, 0, doc_ids_from_lengths(lens)) == \
        sum(n * n for n in lens)


def test_doc_length_generator_golden():
    """The seeded document lengths (seeds 0 and 1) sum to S and stay in [256, 2048]."""
    assert doc_lengths(8192, 0) == [1781, 1398, 1172, 739, 807, 329, 1966]
    assert doc_lengths(8192, 1) == [1104, 1173, 1610, 1960, 318, 2027]
    for seed in range(20):
        lens = doc_lengths(8192, seed)
        assert sum(lens) == 8192 and min(lens) >= 256 and max(lens) <= 2048
