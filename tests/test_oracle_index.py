"""Pins for the oracle's IndexSoftmax attention.

Source: IntAttention (A Fully Integer Attention Pipeline for Efficient Edge
Inference), section 3.1 eqs. 7-10 (row-max distance, quantisation-aligned
clip c_int = round(c sqrt(d) / (s_Q s_K)), index map), section 3.2 (UINT8
exponential table and UINT8 P times 255, integer row sums), the ablation's
(b, c) = (5, 6.6), and eq. 5 for the value path.

Expected values come from closed forms, special cases where the index map
reduces to the identity, an independent series evaluation of the table, and
a bound against the textbook softmax -- never from the oracle itself.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle


def rand_i8(rng, *shape):
    return rng.integers(-127, 128, shape).astype(np.int8)


def exp_series(x: Fraction, terms: int = 60) -> Fraction:
    """e^x by its Taylor series in exact rational arithmetic (|x| <= 8)."""
    s, t = Fraction(1), Fraction(1)
    for n in range(1, terms):
        t = t * x / n
        s += t
    return s


# ------------------------------------------------------------- the table ---

def test_lut_matches_independent_series():
    # LUT[k] = RNE(255 exp(-c k / 31)) for (b, c) = (5, 6.6); the exponential
    # is evaluated here as a rational Taylor series, not with libm.
    lut = oracle.index_lut(6.6, 5)
    assert lut.shape == (32,) and lut.dtype == np.uint8
    c = Fraction(66, 10)
    for k in range(32):
        v = 255 * exp_series(-c * k / 31)
        fl = math.floor(v)
        frac = v - fl
        assert abs(frac - Fraction(1, 2)) > Fraction(1, 1000)   # no near-tie
        want = fl + (1 if frac > Fraction(1, 2) else 0)
        assert int(lut[k]) == want, k


def test_lut_end_points_and_shape():
    lut = oracle.index_lut(6.6, 5)
    assert lut[0] == 255                       # exp(0) -> 255
    assert lut[31] == 0                        # 255 e^-6.6 = 0.348 -> 0
    assert all(lut[k] >= lut[k + 1] for k in range(31))
    for b in (1, 4, 8):
        t = oracle.index_lut(6.6, b)
        assert t.shape == (1 << b,) and t[0] == 255


# --------------------------------------------------------------- c_int ---

def test_cint_closed_forms():
    assert oracle.index_cint(6.6, 64, 1.0, 1.0) == 53       # 6.6 * 8 = 52.8
    assert oracle.index_cint(6.6, 128, 1.0, 1.0) == 75      # 6.6 * 11.3137 = 74.67
    assert oracle.index_cint(6.6, 64, 0.5, 0.25) == 422     # 52.8 / 0.125 = 422.4
    assert oracle.index_cint(6.6, 64, 0.0, 1.0) == 1        # zero scale
    assert oracle.index_cint(6.6, 64, 1e6, 1e6) == 1        # rounds to 0 -> 1


# ------------------------------------------------------------- attention ---

def one_hot_rows(values, d):
    """int8 [n, d] rows with `values` in column 0 and zeros elsewhere."""
    x = np.zeros((len(values), d), np.int8)
    x[:, 0] = values
    return x


def test_identity_index_map():
    # With c_int = 31 and b = 5 the index map floor(D' 31 / c_int) is the
    # identity on D' in [0, 31], so E_j = LUT[min(D_j, 31)] with D_j the
    # integer distance to the row max.  Logits: S_0j = 1 * k_j (column 0).
    d, L = 64, 40
    ks = [40 - j for j in range(L)]        # S = 40, 39, ..., 1 -> D = 0 .. 39
    Qq = one_hot_rows([1] * L, d)
    Kq = one_hot_rows(ks, d)
    Vq = rand_i8(np.random.default_rng(3), L, d)
    sK = np.float32(52.8 / 31)             # c_int = rint(52.8 / sK) = 31
    assert oracle.index_cint(6.6, d, 1.0, float(sK)) == 31
    O, m, l, E = oracle.index_attention_rows(Qq, Kq, Vq, 1.0, float(sK), 0.5, False,
                                             want_stats=True, want_E=True)
    lut = oracle.index_lut(6.6, 5)
    want = [int(lut[min(j, 31)]) for j in range(L)]
    assert list(E[0]) == want
    assert m[0] == 40 and l[0] == sum(want)


def test_halving_index_map():
    # c_int = 62: idx = floor(D / 2) for D <= 62.
    d, L = 64, 30
    ks = [2 * (L - j) for j in range(L)]   # S = 60, 58, ..., 2 -> D = 0, 2, ..., 58
    Qq = one_hot_rows([1] * L, d)
    Kq = one_hot_rows(ks, d)
    Vq = rand_i8(np.random.default_rng(4), L, d)
    sK = np.float32(52.8 / 62)
    assert oracle.index_cint(6.6, d, 1.0, float(sK)) == 62
    _, E = oracle.index_attention_rows(Qq, Kq, Vq, 1.0, float(sK), 1.0, False, want_E=True)
    lut = oracle.index_lut(6.6, 5)
    assert list(E[5]) == [int(lut[(2 * j) // 2]) for j in range(L)]


@pytest.mark.parametrize("causal", [False, True])
def test_constant_logits_give_mean_of_values(causal):
    # Q_hat = 0: every distance is 0, E = 255 for every visible key, so
    # O_i = s_V * mean over visible keys of V_hat.
    rng = np.random.default_rng(5)
    L, d = 33, 128
    Qq = np.zeros((L, d), np.int8)
    Kq, Vq = rand_i8(rng, L, d), rand_i8(rng, L, d)
    O, m, l = oracle.index_attention_rows(Qq, Kq, Vq, 0.03, 0.02, 0.25, causal, want_stats=True)
    for i in range(L):
        n = i + 1 if causal else L
        np.testing.assert_allclose(O[i], 0.25 * Vq[:n].astype(np.float64).mean(axis=0),
                                   rtol=0, atol=1e-12)
        assert l[i] == 255 * n and m[i] == 0


def test_causal_first_row_is_first_value():
    rng = np.random.default_rng(6)
    L, d = 20, 64
    Qq, Kq, Vq = rand_i8(rng, L, d), rand_i8(rng, L, d), rand_i8(rng, L, d)
    O = oracle.index_attention_rows(Qq, Kq, Vq, 0.01, 0.02, 0.5, True)
    np.testing.assert_allclose(O[0], 0.5 * Vq[0].astype(np.float64), rtol=0, atol=1e-12)


def test_two_keys_hand_computed():
    # Row max S = 10, the other key S = 10 - 7 = 3; c_int = 31 -> idx 7.
    d = 64
    Qq = one_hot_rows([1, 1], d)
    Kq = one_hot_rows([10, 3], d)
    Vq = np.zeros((2, d), np.int8)
    Vq[0, :2] = [100, -20]
    Vq[1, :2] = [-50, 80]
    sK = float(np.float32(52.8 / 31))
    sV = float(np.float32(0.1))                      # the scale is an fp32 value
    O = oracle.index_attention_rows(Qq, Kq, Vq, 1.0, sK, sV, False)
    e1 = int(oracle.index_lut(6.6, 5)[7])
    assert e1 == 57                                  # 255 e^{-6.6 * 7 / 31} = 57.39
    for c, (v0, v1) in enumerate([(100, -50), (-20, 80)]):
        assert O[0, c] == pytest.approx(sV * (255 * v0 + e1 * v1) / (255 + e1), abs=1e-12)


@pytest.mark.parametrize("b", [5, 8])
def test_bounded_distance_from_textbook_softmax(b):
    # Per key the weight w = E / 255 lies within the table's bin and rounding
    # error of p = exp(-alpha D) (unclipped keys) or below 255 e^-c / 255 +
    # 0.5 / 255 (clipped keys).  Hence the weighted mean of V_hat moves by at
    # most 2 max|v| sum|w - p| / sum p from the textbook softmax mean, which
    # is computed here with numpy from the integer logits.
    rng = np.random.default_rng(7 + b)
    L, d = 96, 64
    Qq, Kq, Vq = rand_i8(rng, L, d), rand_i8(rng, L, d), rand_i8(rng, L, d)
    sQ, sK, sV = 0.004, 0.005, 0.02
    O = oracle.index_attention_rows(Qq, Kq, Vq, sQ, sK, sV, False, 6.6, b)
    S = Qq.astype(np.int64) @ Kq.astype(np.int64).T
    alpha = np.float64(np.float32(sQ)) * np.float64(np.float32(sK)) / math.sqrt(d)
    cint = oracle.index_cint(6.6, d, sQ, sK)
    lut = oracle.index_lut(6.6, b).astype(np.float64)
    nm1 = (1 << b) - 1
    for i in range(L):
        D = S[i].max() - S[i]
        p = np.exp(-alpha * D)
        ref = sV * (p @ Vq.astype(np.float64)) / p.sum()
        # the table value at each key's bin (recomputed from the clipped index)
        idx = (np.minimum(D, cint) * nm1) // cint
        w = lut[idx] / 255.0
        bound = 2 * 127 * sV * np.abs(w - p).sum() / p.sum()
        assert np.abs(O[i] - ref).max() <= bound + 1e-12
        # and the bin error itself is what the table's resolution allows
        unclipped = D <= cint
        step = math.exp(6.6 / nm1)
        assert np.all(w[unclipped] <= p[unclipped] * step + 0.5 / 255 + 1e-12)
        assert np.all(w[unclipped] >= p[unclipped] - 0.5 / 255 - 1e-12)
