"""Host-side checks of the IndexSoftmax kernel's index arithmetic.

The kernel evaluates idx = floor(D' (2^b - 1) / c_int) (IntAttention section
3.1, eq. 10) as floor(D' q) with q = (2^b - 1) / c_int rounded up to fp32,
through one round-down fma, whenever c_int <= 2^(23 - b).  Both maps are
non-decreasing step functions of the integer D', so they agree everywhere on
[0, c_int] iff they agree at every step of the exact map (its first D' of
each new value, and the D' just before it).  These tests check that, with
exact rational arithmetic, for every b and for c_int up to and at the bound.
"""
from fractions import Fraction

import numpy as np
import pytest


def q_round_up(nm1: int, cint: int) -> Fraction:
    """fp32 (2^b - 1) / c_int rounded toward +infinity, as an exact rational."""
    exact = Fraction(nm1, cint)
    q = np.float32(nm1 / cint)
    if Fraction(float(q)) < exact:
        q = np.nextafter(q, np.float32(np.inf), dtype=np.float32)
    assert Fraction(float(q)) >= exact
    return Fraction(float(q))


def fast_index(dl: int, q: Fraction) -> int:
    # fma.rm(D', q, 2^23) - 2^23 = floor(D' q) while D' q < 2^23
    return int(dl * q // 1)


def check(cint: int, b: int):
    nm1 = (1 << b) - 1
    q = q_round_up(nm1, cint)
    points = {0, cint, cint - 1}
    for k in range(1, nm1 + 1):
        first = -(-k * cint // nm1)          # ceil(k c_int / nm1): first D' with idx >= k
        points.update({first - 1, first, first + 1})
    for dl in points:
        if 0 <= dl <= cint:
            assert fast_index(dl, q) == (dl * nm1) // cint, (cint, b, dl)


@pytest.mark.parametrize("b", range(1, 9))
def test_fast_index_exact_up_to_the_bound(b):
    bound = 1 << (23 - b)
    rng = np.random.default_rng(b)
    cints = list(range(1, 200)) + [bound, bound - 1, bound - 2, bound // 2 + 1]
    cints += [int(x) for x in rng.integers(200, bound, 300)]
    for cint in cints:
        check(cint, b)


def test_fast_index_small_cint_exhaustive():
    for b in (1, 5, 8):
        nm1 = (1 << b) - 1
        for cint in range(1, 300):
            q = q_round_up(nm1, cint)
            for dl in range(cint + 1):
                assert fast_index(dl, q) == (dl * nm1) // cint


def fma_rd_bits(dl: int, q: Fraction) -> int:
    """Bits of fl_down(D' q + 2^23) as fp32 (D' q < 2^23: the value stays in
    [2^23, 2^24), where fp32 has unit spacing)."""
    v = (dl * q + (1 << 23)) // 1
    assert (1 << 23) <= v < (1 << 24)
    return 0x4B000000 + (v - (1 << 23))


@pytest.mark.parametrize("b", [1, 5, 8])
def test_table_address_one_add_stays_in_table(b):
    # The kernel reads entry idx at (base - 0x4B000000) + bits, both mod 2^32,
    # with no clamp: for every visible key (0 <= D' <= c_int) and for a masked
    # key (looked up at D' = 0) the address must land in [base, base + 2^b - 1].
    nm1 = (1 << b) - 1
    rng = np.random.default_rng(40 + b)
    bound = 1 << (23 - b)
    for base in (0, 1024, 0xFFFFF000, int(rng.integers(0, 1 << 32))):
        for cint in [1, 2, 3, nm1, nm1 + 1, bound] + [int(x) for x in rng.integers(1, bound, 20)]:
            q = q_round_up(nm1, cint)
            for dl in {0, 1, cint // 2, cint - 1, cint}:
                if not 0 <= dl <= cint:
                    continue
                addr = ((base - 0x4B000000) + fma_rd_bits(dl, q)) % (1 << 32)
                off = (addr - base) % (1 << 32)
                assert off == (dl * nm1) // cint <= nm1, (base, cint, dl)
