"""Pins of the FP4 oracle (e2m1 code book and encoder, MX block quantiser, Direct-P
attention) against things other than itself: ml_dtypes' e2m1 type, closed forms, the
hand-derived worked examples in tests/golden/fp4_direct_p.json, invariants of the
definition, and a pure-Python brute force on tiny inputs that derives the code boundaries
from the code book's own magnitudes."""
import json
import math
import os

import ml_dtypes
import numpy as np
import pytest

from oracle import fp4

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "fp4_direct_p.json")


def test_code_book_matches_ml_dtypes():
    ref = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(ref, fp4.VALUES)
    assert np.array_equal(np.signbit(ref), np.signbit(fp4.VALUES))


def test_encode_matches_ml_dtypes_cast():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.normal(size=50000) * 3.0,
        rng.uniform(-8, 8, size=50000),
        # exact ties between neighbours, saturation, zeros, tiny values
        [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -5.0, 6.0, 6.5, 7.0, 100.0,
         -100.0, 0.0, -0.0, 1e-30, -1e-30, 0.2500001, 4.9999],
    ]).astype(np.float32)
    got = fp4.encode(x)
    ref = x.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    assert np.array_equal(got, ref)


def test_mx_block_exponent_characterisation():
    """For every nonzero block the stored exponent is the unique X with amax / 2^X in
    [4, 8); a zero block stores -127 and zero codes."""
    rng = np.random.default_rng(1)
    x = rng.normal(size=(6, 256)).astype(np.float32) * np.float32(2.0) ** rng.integers(-20, 20, size=(6, 1))
    x[2, 64:96] = 0.0
    codes, X = fp4.mx_quantize(x)
    amax = np.abs(x.astype(np.float64).reshape(6, 8, 32)).max(axis=2)
    nz = amax > 0
    r = amax[nz] / np.ldexp(1.0, X[nz].astype(np.int64))
    assert np.all((r >= 4.0) & (r < 8.0))
    assert X[2, 2] == -127 and np.all(codes[2, 64:96] & 0x7 == 0)


def test_mx_roundtrip_exact_on_representable_blocks():
    """Values that are e2m1 magnitudes times a common 2^X, with a 4 or a 6 in every block,
    come back exactly."""
    rng = np.random.default_rng(2)
    c = rng.integers(0, 16, size=(4, 128))
    c[:, ::32] = rng.choice([6, 7, 14, 15], size=(4, 4))
    Xs = rng.integers(-30, 30, size=(4, 4))
    x = fp4.VALUES[c] * np.repeat(np.ldexp(1.0, Xs), 32, axis=1)
    codes, X = fp4.mx_quantize(x.astype(np.float32))
    assert np.array_equal(X, Xs)
    assert np.array_equal(fp4.mx_dequantize(codes, X), x)


def test_mx_error_bound_and_axis():
    """|x - x^| <= 2^X (half the widest step) below saturation, and quantising along an
    axis equals quantising the transpose along the last axis."""
    rng = np.random.default_rng(3)
    x = rng.normal(size=(8, 96)).astype(np.float32)
    codes, X = fp4.mx_quantize(x)
    xh = fp4.mx_dequantize(codes, X)
    step = np.repeat(np.ldexp(1.0, X.astype(np.int64)), 32, axis=1)
    a = np.abs(x) / step
    err = np.abs(xh - x)
    assert np.all(err[a <= 6.0] <= step[a <= 6.0])
    assert np.all(np.abs(xh[a > 6.0]) == 6.0 * step[a > 6.0])
    codes_t, X_t = fp4.mx_quantize(x.T, axis=0)
    assert np.array_equal(codes_t, codes.T) and np.array_equal(X_t, X.T)


def test_mx_padding_of_ragged_axis():
    x = np.arange(1, 41, dtype=np.float32)      # 40 values -> two blocks, 24 zeros of padding
    codes, X = fp4.mx_quantize(x)
    assert codes.shape == (64,) and X.shape == (2,)
    assert np.all(codes[40:] == 0)
    xh = fp4.mx_dequantize(codes, X)
    assert xh[39] == 32.0        # 40 / 2^3 = 5 rounds to 4 (ties-to-even not involved)


# ---------------------------------------------------------------- Direct-P


def _half_octave_positions():
    """Positions, in log2 relative to 2^E, that codes 1..7 stand for, derived from the code
    book: the even codes 2, 4, 6 at log2 of their magnitudes (1, 2, 4), each odd code halfway
    between its even neighbours, code 7 half an octave above code 6 and code 1 half an octave
    below code 2."""
    L = {c: math.log2(fp4.VALUES[c]) for c in (2, 4, 6)}
    L[3] = (L[2] + L[4]) / 2
    L[5] = (L[4] + L[6]) / 2
    L[7] = L[6] + (L[6] - L[5])
    L[1] = L[2] - (L[3] - L[2])
    return np.array([L[c] for c in range(1, 8)])


def test_direct_p_codes_at_even_code_magnitudes():
    """A score that sits exactly on the magnitude of code 2, 4 or 6 (relative to E) gets it."""
    for c in (2, 4, 6):
        assert fp4.direct_p_codes(math.log2(fp4.VALUES[c]), 0.0) == c


def test_direct_p_is_nearest_half_octave_position():
    """Brute force over the positions derived from the code book: the code is the nearest
    one; below a quarter octave under code 1's position the code is 0."""
    pos = _half_octave_positions()
    y = np.linspace(-3.0, 2.999, 60001)
    got = fp4.direct_p_codes(y, 0.0)
    d = np.abs(y[:, None] - pos[None, :])
    ref = 1 + np.argmin(d, axis=1)
    ref = np.where(y < pos[0] - (pos[1] - pos[0]) / 2, 0, ref)
    srt = np.sort(d, axis=1)
    clear = (srt[:, 1] - srt[:, 0] > 1e-9) & (np.abs(y - (pos[0] - 0.25)) > 1e-9)
    assert np.array_equal(got[clear], ref[clear])


def test_direct_p_ratio_bound_and_monotone():
    """For codes 2..7 the multiplied magnitude is within [0.75, 1.5 / 2^0.25] of 2^y (the odd
    codes' 1.5 and the saturated top code set the ends); the map is monotone."""
    rng = np.random.default_rng(4)
    y = np.sort(rng.uniform(-0.2499, 3.0, size=100000))
    c = fp4.direct_p_codes(y, 0.0)
    assert np.all(np.diff(c) >= 0) and c.min() >= 2
    ratio = fp4.VALUES[c] / np.exp2(y)
    assert np.all(ratio >= 0.75 - 1e-12)
    assert np.all(ratio <= 1.5 / 2.0 ** 0.25 + 1e-12)
    yy = np.linspace(-20, 3, 5000)
    cc = fp4.direct_p_codes(yy, 0.0)
    assert np.all(np.diff(cc) >= 0) and cc[0] == 0 and cc[-1] == 7


def test_direct_p_integer_shift_scales_exactly():
    """Adding an integer n to every score of a row multiplies P~ by 2^n exactly and leaves
    the codes alone (the block exponent absorbs it)."""
    rng = np.random.default_rng(5)
    t = rng.normal(size=(4, 100)) * 3
    p0, c0, E0 = fp4.direct_p_rows(t)
    for n in (-7, 1, 13):
        p1, c1, E1 = fp4.direct_p_rows(t + n)
        assert np.array_equal(c0, c1) and np.array_equal(E1, E0 + n)
        assert np.array_equal(p1, p0 * 2.0 ** n)


def test_direct_p_block_max_takes_a_top_code():
    rng = np.random.default_rng(6)
    t = rng.normal(size=(8, 256)) * 4
    _, c, _ = fp4.direct_p_rows(t)
    top = c.reshape(8, 8, 32)[np.arange(8)[:, None], np.arange(8)[None, :],
                               np.argmax(t.reshape(8, 8, 32), axis=2)]
    assert np.all((top == 6) | (top == 7))


def test_direct_p_permutation_within_blocks():
    """Permuting keys inside a block (with V alongside) leaves O and LSE unchanged;
    moving a key to another block may not, so only within-block permutations are used."""
    rng = np.random.default_rng(7)
    q = rng.normal(size=(1, 1, 5, 16))
    k = rng.normal(size=(1, 1, 96, 16))
    v = rng.normal(size=(1, 1, 96, 16))
    perm = np.concatenate([rng.permutation(32) + 32 * b for b in range(3)])
    O0, L0 = fp4.attention_fp4_fwd(q, k, v, 0.25)
    O1, L1 = fp4.attention_fp4_fwd(q, k[:, :, perm], v[:, :, perm], 0.25)
    assert np.allclose(O0, O1, rtol=0, atol=1e-12) and np.allclose(L0, L1, rtol=0, atol=1e-12)


def _golden_vectors(case):
    t, v = case["t"], case["v"]
    if isinstance(t, str):                 # "32 x 0.0, then 5.0"
        t = [0.0] * 32 + [5.0]
        v = [[1.0]] * 32 + [[3.0]]
    return np.array(t, dtype=np.float64), np.array(v, dtype=np.float64)


def test_golden_worked_examples():
    with open(GOLDEN) as f:
        cases = json.load(f)["cases"]
    for case in cases:
        t, v = _golden_vectors(case)
        p, c, E = fp4.direct_p_rows(t[None, :])
        assert np.array_equal(E[0], np.array(case["E"], dtype=np.float64)), case["name"]
        if isinstance(case["codes"], list):
            assert np.array_equal(c[0], case["codes"]), case["name"]
            assert np.array_equal(p[0], case["ptilde"]), case["name"]
        # through the attention entry: D = 1, q = 1, k = t, scale = ln 2 (so t is q.k * scale * log2 e)
        q = np.ones((1, 1, 1, 1))
        k = t.reshape(1, 1, -1, 1)
        O, L = fp4.attention_fp4_fwd(q, k, v.reshape(1, 1, -1, 1), math.log(2.0))
        assert abs(O[0, 0, 0, 0] - case["O"][0]) < 1e-12, case["name"]
        assert abs(L[0, 0, 0] - case["LSE"]) < 1e-12, case["name"]


def _brute_force(q, k, v, scale):
    """Pure-Python loops.  Code boundaries come from the code book: halfway between the
    half-octave positions of neighbouring codes (positions from the even codes' magnitudes)."""
    mags = [float(fp4.VALUES[c]) for c in range(8)]
    pos = [float(x) for x in _half_octave_positions()]                             # codes 1..7
    bounds = [pos[0] - (pos[1] - pos[0]) / 2] + [(pos[c] + pos[c + 1]) / 2 for c in range(6)]
    Sq, D = len(q), len(q[0])
    Sk = len(k)
    out, lse = [], []
    for i in range(Sq):
        t = [sum(q[i][d] * k[j][d] for d in range(D)) * scale / math.log(2.0) for j in range(Sk)]
        w = [0.0] * Sk
        for b0 in range(0, Sk, 32):
            blk = range(b0, min(b0 + 32, Sk))
            E = math.floor(max(t[j] for j in blk)) - 2
            for j in blk:
                y = t[j] - E
                code = sum(1 for bd in bounds if y >= bd)
                w[j] = mags[code] * 2.0 ** E
        s = sum(w)
        out.append([sum(w[j] * v[j][d] for j in range(Sk)) / s for d in range(D)])
        lse.append(math.log(s))
    return out, lse


@pytest.mark.parametrize("Sq,Sk,D,mul", [(3, 70, 8, 1.0), (2, 33, 4, 4.0), (4, 5, 3, 0.3)])
def test_attention_matches_brute_force(Sq, Sk, D, mul):
    rng = np.random.default_rng(Sq * 100 + Sk)
    q = rng.normal(size=(Sq, D)) * mul
    k = rng.normal(size=(Sk, D))
    v = rng.normal(size=(Sk, D))
    scale = 1.0 / math.sqrt(D)
    O_bf, L_bf = _brute_force(q.tolist(), k.tolist(), v.tolist(), scale)
    O, L = fp4.attention_fp4_fwd(q[None, None], k[None, None], v[None, None], scale)
    assert np.allclose(O[0, 0], np.array(O_bf), rtol=0, atol=1e-12)
    assert np.allclose(L[0, 0], np.array(L_bf), rtol=0, atol=1e-12)


def test_attention_equal_scores_give_the_mean():
    rng = np.random.default_rng(8)
    v = rng.normal(size=(1, 1, 77, 8))
    k = np.zeros((1, 1, 77, 8))
    q = rng.normal(size=(1, 1, 3, 8))
    O, L = fp4.attention_fp4_fwd(q, k, v, 0.3)
    assert np.allclose(O[0, 0], np.broadcast_to(v[0, 0].mean(axis=0), (3, 8)), rtol=0, atol=1e-12)
    # t = 0 everywhere: E = -2, code 6 (magnitude 4), P~ = 1 per key
    assert np.allclose(L, math.log(77.0), rtol=0, atol=1e-12)


def test_attention_grouped_heads_read_their_kv_head():
    rng = np.random.default_rng(9)
    q = rng.normal(size=(1, 4, 3, 8))
    k = rng.normal(size=(1, 2, 40, 8))
    v = rng.normal(size=(1, 2, 40, 8))
    O, L = fp4.attention_fp4_fwd(q, k, v, 0.35)
    for h in range(4):
        Oh, Lh = fp4.attention_fp4_fwd(q[:, h:h + 1], k[:, h // 2:h // 2 + 1], v[:, h // 2:h // 2 + 1], 0.35)
        assert np.array_equal(O[:, h], Oh[:, 0]) and np.array_equal(L[:, h], Lh[:, 0])
