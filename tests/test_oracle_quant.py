"""Pins for the oracle's quantiser (IntAttention, section 2.1, eq. 3:
s_X = max|X| / 127, X ~= s_X X_hat, zero-point 0; per-token rows for Q/K per
INT-FlashAttention's abstract, one scale per L x d tensor for V).

Every expected value here comes from a closed form or from exact rational
arithmetic written in this file, never from the oracle itself.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle


def fl32(r: Fraction) -> Fraction:
    """Round a rational to the nearest IEEE binary32 value, ties to even
    (normal range only), in exact arithmetic."""
    if r == 0:
        return Fraction(0)
    sign = -1 if r < 0 else 1
    a = abs(r)
    e = 0
    while a >= 2:
        a /= 2
        e += 1
    while a < 1:
        a *= 2
        e -= 1
    m = a * (1 << 23)                 # in [2^23, 2^24)
    lo = m.numerator // m.denominator
    rem = m - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return sign * Fraction(lo) * Fraction(2) ** (e - 23)


def rne(r: Fraction) -> int:
    """Round to nearest integer, ties to even (exact)."""
    fl = r.numerator // r.denominator
    rem = r - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return int(fl)


def expected_codes(row):
    """Eq. 3 with IEEE fp32 s = fl(amax / 127) and fl(x / s), then RNE and the
    symmetric clamp, computed exactly."""
    amax = max(abs(Fraction(float(v))) for v in row)
    s = fl32(amax / 127)
    if s == 0:
        return [0] * len(row), 0.0
    codes = [max(-127, min(127, rne(fl32(Fraction(float(v)) / s)))) for v in row]
    return codes, float(s)


def test_unit_scale_closed_form_ties_to_even():
    # amax = 127 gives s = 1 exactly, so x_hat = RNE(x): ties go to even.
    row = np.array([127.0, 2.5, -3.5, 0.5, 1.5, -0.5, 126.5, -2.25, 0.0], np.float32)
    q, s = oracle.quantize_per_token(row[None, :])
    assert s[0] == 1.0
    assert q[0].tolist() == [127, 2, -4, 0, 2, 0, 126, -2, 0]


def test_half_scale_closed_form():
    # amax = 63.5 gives s = 0.5 exactly, so x_hat = RNE(2 x).
    row = np.array([63.5, 1.25, -1.25, 0.75, 0.25, -63.5], np.float32)
    q, s = oracle.quantize_per_token(row[None, :])
    assert s[0] == 0.5
    assert q[0].tolist() == [127, 2, -2, 2, 0, -127]


def test_matches_exact_ieee_division_on_random_fp16_rows():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((64, 128)).astype(np.float16).astype(np.float32)
    q, s = oracle.quantize_per_token(x)
    for r in range(x.shape[0]):
        codes, sr = expected_codes(x[r])
        assert s[r] == np.float32(sr)
        assert q[r].tolist() == codes


def test_division_not_reciprocal_multiply():
    # Find fp16 pairs (amax, x) whose code depends on computing fl(x / s)
    # rather than x * fl(1 / s); the exact-arithmetic rule must win on all.
    allh = np.arange(1, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float32)
    rng = np.random.default_rng(7)
    amaxes = np.unique(rng.choice(allh[(allh > 0.1) & (allh < 100)], 400))
    rows = []
    for a in amaxes:
        s = np.float32(a / np.float32(127.0))
        x = allh[allh <= a]
        hard = x[np.rint(x / s) != np.rint(x * (np.float32(1.0) / s))]
        rows += [[a, h] for h in hard[:2]]
    assert len(rows) >= 20, "too few discriminating inputs found"
    x = np.array(rows, np.float32)
    q, sq = oracle.quantize_per_token(x)
    for r in range(x.shape[0]):
        codes, sr = expected_codes(x[r])
        assert sq[r] == np.float32(sr)
        assert q[r].tolist() == codes


def test_round_trip_bound_and_range():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((256, 64)) * rng.uniform(0.01, 50, (256, 1))).astype(np.float16)
    x = x.astype(np.float32)
    q, s = oracle.quantize_per_token(x)
    assert np.abs(q.astype(np.int32)).max() <= 127
    err = np.abs(x.astype(np.float64) - s[:, None].astype(np.float64) * q)
    # |x - s x_hat| <= s/2 plus the fp32 rounding of the quotient (<= 127 * 2^-24 codes)
    assert np.all(err <= s[:, None] * (0.5 + 127 * 2.0 ** -24) + 1e-30)
    # the element of largest magnitude maps to +-127
    am = np.abs(x).argmax(axis=1)
    picked = q[np.arange(x.shape[0]), am].astype(np.int32)
    assert np.all(np.abs(picked) == 127)
    assert np.all(np.sign(picked) == np.sign(x[np.arange(x.shape[0]), am]))


def test_sign_symmetry_and_power_of_two_invariance():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((32, 128)).astype(np.float16).astype(np.float32)
    q, s = oracle.quantize_per_token(x)
    qn, sn = oracle.quantize_per_token(-x)
    assert np.array_equal(qn, -q) and np.array_equal(sn, s)
    q4, s4 = oracle.quantize_per_token(x * 4)
    assert np.array_equal(q4, q) and np.array_equal(s4, s * 4)


def test_zero_rows_and_on_grid_inputs_are_lossless():
    x = np.zeros((3, 64), np.float32)
    q, s = oracle.quantize_per_token(x)
    assert not q.any() and not s.any()
    # x = s k with s a power of two and a +-127 in every row: quantisation is exact
    rng = np.random.default_rng(4)
    k = rng.integers(-127, 128, (16, 64))
    k[:, 5] = 127 * np.where(rng.integers(0, 2, 16) == 0, -1, 1)
    sc = 2.0 ** -5
    q, s = oracle.quantize_per_token((k * sc).astype(np.float32))
    assert np.all(s == sc) and np.array_equal(q.astype(np.int64), k)


@pytest.mark.parametrize("groups", [1, 3])
def test_per_tensor_one_scale_per_group(groups):
    rng = np.random.default_rng(5)
    x = rng.standard_normal((groups, 40, 64)).astype(np.float16).astype(np.float32)
    x[-1, 7, 9] = 9.0  # a large value in the last group only
    q, s = oracle.quantize_per_tensor(x, groups)
    for g in range(groups):
        codes, sg = expected_codes(x[g].ravel())
        assert s[g] == np.float32(sg)
        assert q[g].ravel().tolist() == codes
    assert s[-1] == np.float32(fl32(Fraction(9) / 127))


# ------------------------------------------------ b-bit codes (INT4 remark) ---

def test_bits8_is_the_int8_quantiser():
    rng = np.random.default_rng(31)
    x = (rng.standard_normal((50, 128)) * 3).astype(np.float16).astype(np.float32)
    q8, s8 = oracle.quantize_per_token(x)
    qb, sb = oracle.quantize_per_token_bits(x, 8)
    np.testing.assert_array_equal(q8, qb)
    np.testing.assert_array_equal(s8.view(np.uint32), sb.view(np.uint32))


def test_bits4_hand_table():
    # x = [1, -0.5, 0.25, 0.07]: s = fl32(1/7) = 0.142857149... (above 1/7), so
    # -0.5/s = -3.4999998 in fp32 (no tie) -> -3; 0.25/s = 1.7499999 -> 2;
    # 0.07/s = 0.49 -> 0; 1/s rounds to 7
    x = np.array([[1.0, -0.5, 0.25, 0.07, 0, 0, 0, 0]], np.float32)
    q, s = oracle.quantize_per_token_bits(x, 4)
    assert s[0] == np.float32(1.0) / np.float32(7.0)
    assert list(q[0, :4]) == [7, -3, 2, 0]
    # a genuine tie: 0.5 with s = 1/4 exactly (amax 1.75 = 7/4): 0.5/0.25 = 2.0,
    # 0.625/0.25 = 2.5 -> 2 (even), 0.875/0.25 = 3.5 -> 4 (even)
    y = np.array([[1.75, 0.5, 0.625, 0.875, 0, 0, 0, 0]], np.float32)
    q, s = oracle.quantize_per_token_bits(y, 4)
    assert s[0] == np.float32(0.25)
    assert list(q[0, :4]) == [7, 2, 2, 4]


@pytest.mark.parametrize("bits", [2, 3, 4, 6])
def test_bits_round_trip_and_range(bits):
    rng = np.random.default_rng(bits)
    x = (rng.standard_normal((40, 64)) * 2).astype(np.float16).astype(np.float32)
    q, s = oracle.quantize_per_token_bits(x, bits)
    qmax = (1 << (bits - 1)) - 1
    assert np.abs(q).max() <= qmax
    assert np.all(np.abs(q).max(axis=1) == qmax)            # the arg-max row entry hits +-qmax
    err = np.abs(x - s[:, None].astype(np.float64) * q)
    assert np.all(err <= s[:, None] / 2 * (1 + 1e-6) + 1e-12)


@pytest.mark.parametrize("amax", [127.0, 100.0, 1.0, 0.0999755859375, 3.0517578125e-05])
def test_near_ties_against_exact_rational(amax):
    """Every fp16 x whose fp32 quotient x / s lies within 2e-3 of a
    half-integer (the elements the GPU kernels send to the IEEE division,
    and the exact ties), both signs, in one row with the row's maximum: the
    oracle's codes equal RNE(fl32(x / s)) computed in exact arithmetic."""
    h = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float32)
    h = h[h <= np.float32(amax)]
    s32 = np.float32(np.float32(amax) / np.float32(127.0))
    q = h / s32
    near = h[np.abs(q - np.floor(q) - np.float32(0.5)) < np.float32(2e-3)]
    assert near.size > 0
    row = np.concatenate([[np.float32(amax)], near, -near]).astype(np.float32)
    codes, s = expected_codes(row)
    qo, so = oracle.quantize_per_token(row[None, :])
    assert so[0] == np.float32(s)
    np.testing.assert_array_equal(qo[0], np.array(codes, np.int8))
