"""Pins for the oracle's decode function (one query against a key / value
cache, keys cut into ranges that each run the online steps, merged at the
end).  Sources: INT-FlashAttention abstract and FlashAttention-3 abstract
(the block-wise online form), IntAttention eqs. 4-5 and section 3.2.

Expected values come from the independently pinned online attention on the
same rows, closed forms, and integer logits computed with numpy."""
import math

import numpy as np
import pytest

import oracle


def rand_i8(rng, *shape):
    return rng.integers(-127, 128, shape).astype(np.int8)


def online_last_row(q, sq, Kq, sK, Vq, sV):
    """The online oracle's answer for a query placed as the last row of a
    non-causal problem over these keys, and its row sum."""
    L, d = Kq.shape
    Qq = np.zeros((L, d), np.int8)
    Qq[-1] = q
    sQ = np.ones(L, np.float32)
    sQ[-1] = sq
    O, l = oracle.attention_online_rows(Qq, Kq, Vq, sQ, sK, sV, False, 128, L - 1, L, want_l=True)
    return O[0], l[0]


@pytest.mark.parametrize("L,d", [(300, 64), (1000, 128), (128, 128), (1, 64)])
def test_one_range_is_the_online_row(L, d):
    rng = np.random.default_rng(L + d)
    q, Kq, Vq = rand_i8(rng, d), rand_i8(rng, L, d), rand_i8(rng, L, d)
    sK = rng.uniform(0.005, 0.02, L).astype(np.float32)
    sq, sV = np.float32(0.013), np.float32(0.02)
    O = oracle.decode(q, sq, Kq, sK, Vq, sV)
    want, _ = online_last_row(q, sq, Kq, sK, Vq, sV)
    np.testing.assert_allclose(O, want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("split_len", [128, 256, 1024])
def test_constant_logits_mean_of_values(split_len):
    rng = np.random.default_rng(5)
    L, d = 700, 128
    q = np.zeros(d, np.int8)
    Kq, Vq = rand_i8(rng, L, d), rand_i8(rng, L, d)
    sK = rng.uniform(0.005, 0.02, L).astype(np.float32)
    O = oracle.decode(q, 0.01, Kq, sK, Vq, 0.25, 128, split_len)
    np.testing.assert_allclose(O, 0.25 * Vq.astype(np.float64).mean(axis=0), rtol=0, atol=1e-12)


def test_two_ranges_merge_the_range_results():
    # keys [0, 256) and [256, 400) as two ranges: each range's result is the
    # online oracle on that range alone; the merge weights each range by its
    # row sum times e^(m_s - M), with m_s from integer logits.
    rng = np.random.default_rng(9)
    L, d, split = 400, 64, 256
    q, Kq, Vq = rand_i8(rng, d), rand_i8(rng, L, d), rand_i8(rng, L, d)
    sK = rng.uniform(0.005, 0.02, L).astype(np.float32)
    sq, sV = np.float32(0.02), np.float32(0.03)
    O = oracle.decode(q, sq, Kq, sK, Vq, sV, 128, split)
    parts = []
    for r0, r1 in [(0, split), (split, L)]:
        Os, ls = online_last_row(q, sq, Kq[r0:r1], sK[r0:r1], Vq[r0:r1], sV)
        S = Kq[r0:r1].astype(np.int64) @ q.astype(np.int64)
        t = S * np.float64(sq) * sK[r0:r1].astype(np.float64) / math.sqrt(d)
        parts.append((t.max(), ls, Os))
    M = max(p[0] for p in parts)
    num = sum(math.exp(m - M) * l * Os for m, l, Os in parts)
    den = sum(math.exp(m - M) * l for m, l, _ in parts)
    np.testing.assert_allclose(O, num / den, rtol=1e-12, atol=1e-12)
