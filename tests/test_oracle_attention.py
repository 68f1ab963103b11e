"""Pins for the oracle's integer logits and quantised attention.

Sources: IntAttention (A Fully Integer Attention Pipeline for Efficient Edge
Inference) section 2.1 eq. 1 (attention), eq. 4 (INT8 x INT8 -> INT32 logits,
alpha = s_Q s_K / sqrt(d) as section 3.1 eq. 8 spells out), eq. 5
(O ~= s_V P V_hat), section 2.2 eq. 6 (row-max-stable softmax) and section
3.2 (P x 127 stored as INT8).

Expected values come from closed forms, special cases, hand-built inputs with
known logits, or brute-force loops on tiny inputs -- never from the oracle.
"""
import math

import numpy as np
import pytest

import oracle


def rand_i8(rng, *shape):
    return rng.integers(-127, 128, shape).astype(np.int8)


# ---------------------------------------------------------------- Q K^T ---

@pytest.mark.parametrize("d", [64, 128])
def test_qk_int32_brute_force(d):
    rng = np.random.default_rng(10 + d)
    Qq, Kq = rand_i8(rng, 2, 5, d), rand_i8(rng, 2, 5, d)
    S = oracle.qk_int32(Qq, Kq)
    for h in range(2):
        for i in range(5):
            for j in range(5):
                want = 0
                for k in range(d):
                    want += int(Qq[h, i, k]) * int(Kq[h, j, k])
                assert S[h, i, j] == want


@pytest.mark.parametrize("d", [64, 128])
def test_qk_int32_extremes(d):
    Qq = np.full((1, 2, d), 127, np.int8)
    Kq = np.full((1, 2, d), 127, np.int8)
    Kq[0, 1] = -127
    S = oracle.qk_int32(Qq, Kq)
    assert S[0, 0, 0] == 127 * 127 * d and S[0, 0, 1] == -127 * 127 * d


# ----------------------------------------------------- quantised attention ---

@pytest.mark.parametrize("causal", [False, True])
def test_constant_logits_give_mean_of_values(causal):
    # Q_hat = 0: every logit is 0, p = 1, every P code is 127, so
    # O_i = s_V * mean over visible keys of V_hat (exact up to fp64 rounding).
    rng = np.random.default_rng(11)
    L, d = 37, 64
    Qq = np.zeros((L, d), np.int8)
    Kq, Vq = rand_i8(rng, L, d), rand_i8(rng, L, d)
    sQ = rng.uniform(0.01, 0.1, L).astype(np.float32)
    sK = rng.uniform(0.01, 0.1, L).astype(np.float32)
    sV = 0.037
    O, m, l, P = oracle.attention_rows(Qq, Kq, Vq, sQ, sK, sV, causal, want_stats=True, want_P=True)
    for i in range(L):
        n = i + 1 if causal else L
        want = np.float32(sV) * Vq[:n].astype(np.float64).mean(axis=0)
        np.testing.assert_allclose(O[i], want, rtol=1e-13, atol=1e-15)
        assert m[i] == 0.0 and l[i] == n
        assert np.all(P[i, :n] == 127) and np.all(P[i, n:] == 0)


def test_causal_first_row_is_first_value():
    rng = np.random.default_rng(12)
    L, d = 9, 128
    Qq, Kq, Vq = rand_i8(rng, L, d), rand_i8(rng, L, d), rand_i8(rng, L, d)
    s = rng.uniform(0.01, 0.1, L).astype(np.float32)
    O = oracle.attention_rows(Qq, Kq, Vq, s, s, 0.5, True)
    np.testing.assert_array_equal(O[0], 0.5 * Vq[0].astype(np.float64))


@pytest.mark.parametrize("d", [64, 128])
def test_hand_built_logits(d):
    # Q_hat row 0 = a e_0, K_hat row j = b_j e_0, so S_0j = a b_j exactly and
    # t_j = a b_j s_Q s_K[j] / sqrt(d); the rest follows eq. 6, section 3.2 and eq. 5.
    a, b = 100, [127, 50, -127, 0, 90]
    L = len(b)
    Qq = np.zeros((L, d), np.int8)
    Qq[0, 0] = a
    Kq = np.zeros((L, d), np.int8)
    Kq[:, 0] = b
    rng = np.random.default_rng(13)
    Vq = rand_i8(rng, L, d)
    sQ = np.full(L, 0.03125, np.float32)
    sK = np.array([0.02, 0.05, 0.01, 0.07, 0.04], np.float32)
    sV = 0.02
    O, m, l, P = oracle.attention_rows(Qq, Kq, Vq, sQ, sK, sV, False, 0, 1,
                                       want_stats=True, want_P=True)
    t = [a * b[j] * float(sQ[0]) * float(sK[j]) / math.sqrt(d) for j in range(L)]
    mx = max(t)
    p = [math.exp(tj - mx) for tj in t]
    codes = [round(127 * pj) for pj in p]   # Python round: ties to even
    assert P[0].tolist() == codes
    assert m[0] == pytest.approx(mx, rel=1e-15)
    assert l[0] == pytest.approx(sum(p), rel=1e-15)
    want = [float(np.float32(sV)) * sum(codes[j] * int(Vq[j, c]) for j in range(L)) / (127 * sum(p))
            for c in range(d)]
    np.testing.assert_allclose(O[0], want, rtol=1e-13)


def test_causal_rows_ignore_future_keys():
    rng = np.random.default_rng(14)
    L, d = 20, 64
    Qq, Kq, Vq = rand_i8(rng, L, d), rand_i8(rng, L, d), rand_i8(rng, L, d)
    sQ = rng.uniform(0.005, 0.05, L).astype(np.float32)
    sK = rng.uniform(0.005, 0.05, L).astype(np.float32)
    O1 = oracle.attention_rows(Qq, Kq, Vq, sQ, sK, 0.03, True)
    K2, V2, sK2 = Kq.copy(), Vq.copy(), sK.copy()
    K2[12:] = rand_i8(rng, L - 12, d)
    V2[12:] = rand_i8(rng, L - 12, d)
    sK2[12:] *= 3
    O2 = oracle.attention_rows(Qq, K2, V2, sQ, sK2, 0.03, True)
    np.testing.assert_array_equal(O1[:12], O2[:12])
    assert not np.array_equal(O1[12:], O2[12:])


def test_p_codes_range_and_argmax():
    rng = np.random.default_rng(15)
    L, d = 50, 128
    Qq, Kq, Vq = rand_i8(rng, L, d), rand_i8(rng, L, d), rand_i8(rng, L, d)
    sQ = rng.uniform(0.005, 0.05, L).astype(np.float32)
    sK = rng.uniform(0.005, 0.05, L).astype(np.float32)
    _, m, l, P = oracle.attention_rows(Qq, Kq, Vq, sQ, sK, 0.03, False, want_stats=True, want_P=True)
    S = Qq.astype(np.int64) @ Kq.astype(np.int64).T
    t = S * sQ[:, None].astype(np.float64) * sK[None, :].astype(np.float64) / math.sqrt(d)
    assert P.min() >= 0 and P.max() == 127
    for i in range(L):
        assert P[i, np.argmax(t[i])] == 127
        order = np.argsort(t[i])
        assert np.all(np.diff(P[i, order]) >= 0)   # codes are monotone in the logit
        assert 1.0 <= l[i] <= L


def test_on_grid_inputs_error_is_only_p_rounding():
    # Q, K, V exactly on the INT8 grid (power-of-two scales, a +-127 per row):
    # quantisation is lossless, so the gap to fp64 attention comes from the P
    # codes alone: |O - O_ref| <= 0.5 s_V n max|V_hat| / (127 l).
    rng = np.random.default_rng(16)
    L, d = 64, 64
    def grid(sc):
        k = rng.integers(-127, 128, (L, d))
        k[:, 3] = 127
        return k, (k * sc).astype(np.float32)
    kq, Q = grid(2.0 ** -6)
    kk, K = grid(2.0 ** -6)
    kv, V = grid(2.0 ** -5)
    V = V.copy()
    Qq, sQ = oracle.quantize_per_token(Q)
    Kq, sK = oracle.quantize_per_token(K)
    Vq, sV = oracle.quantize_per_tensor(V, 1)
    assert np.array_equal(Qq.astype(np.int64), kq) and np.array_equal(Vq.astype(np.int64), kv)
    for causal in (False, True):
        O, m, l = oracle.attention_rows(Qq, Kq, Vq, sQ, sK, float(sV[0]), causal, want_stats=True)
        ref = oracle.attention_fp64_rows(Q, K, V, causal)
        n = (np.arange(L) + 1) if causal else np.full(L, L)
        bound = 0.5 * float(sV[0]) * n * 127 / (127 * l)
        assert np.all(np.abs(O - ref).max(axis=1) <= bound * (1 + 1e-9))


# ------------------------------------------------------ fp64 reference ---

def test_fp64_brute_force_tiny():
    rng = np.random.default_rng(17)
    L, d = 4, 3
    Q, K, V = (rng.standard_normal((L, d)).astype(np.float32) for _ in range(3))
    for causal in (False, True):
        O = oracle.attention_fp64_rows(Q, K, V, causal)
        for i in range(L):
            n = i + 1 if causal else L
            a = [sum(float(Q[i, k]) * float(K[j, k]) for k in range(d)) / math.sqrt(d) for j in range(n)]
            w = [math.exp(x) for x in a]
            z = sum(w)
            for c in range(d):
                assert O[i, c] == pytest.approx(sum(w[j] * float(V[j, c]) for j in range(n)) / z,
                                                rel=1e-12, abs=1e-14)


def test_fp64_special_cases():
    rng = np.random.default_rng(18)
    L, d = 16, 64
    K, V = (rng.standard_normal((L, d)).astype(np.float32) for _ in range(2))
    Q = np.zeros((L, d), np.float32)
    O = oracle.attention_fp64_rows(Q, K, V, False)
    np.testing.assert_allclose(O, np.broadcast_to(V.astype(np.float64).mean(0), (L, d)), rtol=1e-12, atol=1e-14)
    Q = rng.standard_normal((L, d)).astype(np.float32)
    O = oracle.attention_fp64_rows(Q, K, V, True)
    np.testing.assert_array_equal(O[0], V[0].astype(np.float64))


# ------------------------------------------------ block-wise online form ---

@pytest.mark.parametrize("causal", [False, True])
def test_online_single_block_equals_two_pass(causal):
    # One block of keys: the running max is the final max, so the online form
    # performs exactly the two-pass arithmetic.
    rng = np.random.default_rng(20)
    L, d = 100, 64
    Qq, Kq, Vq = rand_i8(rng, L, d), rand_i8(rng, L, d), rand_i8(rng, L, d)
    sQ = rng.uniform(0.005, 0.05, L).astype(np.float32)
    sK = rng.uniform(0.005, 0.05, L).astype(np.float32)
    O2 = oracle.attention_rows(Qq, Kq, Vq, sQ, sK, 0.03, causal)
    O1 = oracle.attention_online_rows(Qq, Kq, Vq, sQ, sK, 0.03, causal, block=128)
    np.testing.assert_array_equal(O1, O2)


def test_online_equals_two_pass_when_max_is_in_first_block():
    # Key 0 is aligned with every query and much larger than the rest: the
    # running max is final after the first block, alpha = 1 afterwards and the
    # block sums add up to the two-pass integer sum exactly (only the order of
    # the fp64 row-sum additions differs).
    rng = np.random.default_rng(21)
    L, d = 300, 128
    Qq = rng.integers(1, 128, (L, d)).astype(np.int8)
    Kq = rng.integers(-20, 21, (L, d)).astype(np.int8)
    Kq[0] = 127
    Vq = rand_i8(rng, L, d)
    sQ = rng.uniform(0.005, 0.02, L).astype(np.float32)
    sK = np.full(L, 0.01, np.float32)
    for causal in (False, True):
        O2 = oracle.attention_rows(Qq, Kq, Vq, sQ, sK, 0.03, causal)
        for block in (16, 64, 128):
            O1 = oracle.attention_online_rows(Qq, Kq, Vq, sQ, sK, 0.03, causal, block=block)
            np.testing.assert_allclose(O1, O2, rtol=1e-13, atol=0)


def test_online_hand_built_two_blocks():
    # block = 2, keys with logits [0, 1 | 3, 2] (row 0): the P codes of the
    # first block are taken against m = 1, rescaled by e^(1 - 3) when block 2
    # raises the max to 3 (FlashAttention's running max / running sum).
    d = 64
    a, b = 64, [0, 1, 3, 2]                 # S_0j = a b_j; t_j = a b_j sQ sK / 8 = b_j
    L = len(b)
    Qq = np.zeros((L, d), np.int8)
    Qq[0, 0] = a
    Kq = np.zeros((L, d), np.int8)
    Kq[:, 0] = b
    sQ = np.full(L, 0.125, np.float32)
    sK = np.full(L, 1.0, np.float32)
    rng = np.random.default_rng(22)
    Vq = rand_i8(rng, L, d)
    O, l = oracle.attention_online_rows(Qq, Kq, Vq, sQ, sK, 0.5, False, block=2, r0=0, r1=1,
                                        want_l=True)
    c1 = [round(127 * math.exp(t - 1)) for t in (0, 1)]
    c2 = [round(127 * math.exp(t - 3)) for t in (3, 2)]
    alpha = math.exp(1 - 3)
    acc = [alpha * (c1[0] * int(Vq[0, c]) + c1[1] * int(Vq[1, c])) + (c2[0] * int(Vq[2, c]) + c2[1] * int(Vq[3, c]))
           for c in range(d)]
    lw = alpha * (math.exp(-1) + 1) + (1 + math.exp(-1))
    assert l[0] == pytest.approx(lw, rel=1e-15)
    np.testing.assert_allclose(O[0], [0.5 * x / (127 * lw) for x in acc], rtol=1e-13)
    # and the two-pass form takes all four codes against m = 3
    O2 = oracle.attention_rows(Qq, Kq, Vq, sQ, sK, 0.5, False, 0, 1)
    c = [round(127 * math.exp(t - 3)) for t in b]
    want = [0.5 * sum(c[j] * int(Vq[j, k]) for j in range(4)) / (127 * sum(math.exp(t - 3) for t in b))
            for k in range(d)]
    np.testing.assert_allclose(O2[0], want, rtol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_online_constant_logits(causal):
    rng = np.random.default_rng(23)
    L, d = 300, 64
    Qq = np.zeros((L, d), np.int8)
    Kq, Vq = rand_i8(rng, L, d), rand_i8(rng, L, d)
    s = rng.uniform(0.01, 0.1, L).astype(np.float32)
    O = oracle.attention_online_rows(Qq, Kq, Vq, s, s, 0.25, causal, block=128)
    for i in range(L):
        n = i + 1 if causal else L
        np.testing.assert_allclose(O[i], 0.25 * Vq[:n].astype(np.float64).mean(0), rtol=1e-13, atol=1e-15)


# ------------------------------------------ row sum from the P codes (f3) ---

@pytest.mark.parametrize("causal", [False, True])
def test_codesum_constant_logits_give_mean_of_values(causal):
    # Q_hat = 0: every code is 127, so sum codes / 127 = the number of keys and
    # O is the mean of the visible V_hat rows, as with the p-sum
    rng = np.random.default_rng(21)
    L, d = 200, 64
    Qq = np.zeros((L, d), np.int8)
    Kq, Vq = rand_i8(rng, L, d), rand_i8(rng, L, d)
    sQ = rng.uniform(0.01, 0.1, L).astype(np.float32)
    sK = rng.uniform(0.01, 0.1, L).astype(np.float32)
    O = oracle.attention_online_rows(Qq, Kq, Vq, sQ, sK, 0.5, causal, 128, lsum_codes=True)
    for i in range(L):
        n = i + 1 if causal else L
        np.testing.assert_allclose(O[i], 0.5 * Vq[:n].astype(np.float64).mean(axis=0), rtol=0, atol=1e-12)


def test_codesum_one_block_is_the_code_weighted_mean():
    # one key block: the online form is the two-pass form, and with the row
    # sum taken from the codes O_i = s_V sum_j P_ij V_j / sum_j P_ij exactly,
    # with the P codes of the (separately pinned) two-pass function
    rng = np.random.default_rng(22)
    L, d = 100, 128
    Qq, Kq, Vq = rand_i8(rng, L, d), rand_i8(rng, L, d), rand_i8(rng, L, d)
    sQ = rng.uniform(0.002, 0.01, L).astype(np.float32)
    sK = rng.uniform(0.002, 0.01, L).astype(np.float32)
    sV = float(np.float32(0.03))
    _, P = oracle.attention_rows(Qq, Kq, Vq, sQ, sK, sV, False, want_P=True)
    O = oracle.attention_online_rows(Qq, Kq, Vq, sQ, sK, sV, False, 128, lsum_codes=True)
    want = sV * (P.astype(np.float64) @ Vq.astype(np.float64)) / P.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(O, want, rtol=1e-12, atol=1e-12)


# ------------------------------- UINT8 P codes, RNE(255 p) (Table 5 scheme) ---

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("lsum_codes", [False, True])
def test_uint8_p_constant_logits_give_mean_of_values(causal, lsum_codes):
    # Q_hat = 0: every p is 1, every code 255; O is the mean of the visible V_hat
    rng = np.random.default_rng(31)
    L, d = 260, 64
    Qq = np.zeros((L, d), np.int8)
    Kq, Vq = rand_i8(rng, L, d), rand_i8(rng, L, d)
    s = rng.uniform(0.01, 0.1, L).astype(np.float32)
    O = oracle.attention_online_rows(Qq, Kq, Vq, s, s, 0.25, causal, 128, lsum_codes=lsum_codes,
                                     p_levels=255)
    for i in range(L):
        n = i + 1 if causal else L
        np.testing.assert_allclose(O[i], 0.25 * Vq[:n].astype(np.float64).mean(0), rtol=1e-13, atol=1e-15)


def test_uint8_p_hand_built_two_blocks():
    # the two-block example with 255 levels: codes RNE(255 e^(t - m)) against
    # the running max (1, then 3), acc and l rescaled by e^(1 - 3)
    d = 64
    a, b = 64, [0, 1, 3, 2]                 # t_j = a b_j sQ sK / 8 = b_j
    L = len(b)
    Qq = np.zeros((L, d), np.int8)
    Qq[0, 0] = a
    Kq = np.zeros((L, d), np.int8)
    Kq[:, 0] = b
    sQ = np.full(L, 0.125, np.float32)
    sK = np.full(L, 1.0, np.float32)
    rng = np.random.default_rng(32)
    Vq = rand_i8(rng, L, d)
    c1 = [round(255 * math.exp(t - 1)) for t in (0, 1)]     # [94, 255]
    c2 = [round(255 * math.exp(t - 3)) for t in (3, 2)]     # [255, 94]
    assert c1 == [94, 255] and c2 == [255, 94]
    alpha = math.exp(1 - 3)
    acc = [alpha * (c1[0] * int(Vq[0, c]) + c1[1] * int(Vq[1, c])) + (c2[0] * int(Vq[2, c]) + c2[1] * int(Vq[3, c]))
           for c in range(d)]
    for lsum_codes in (False, True):
        O, l = oracle.attention_online_rows(Qq, Kq, Vq, sQ, sK, 0.5, False, block=2, r0=0, r1=1,
                                            want_l=True, lsum_codes=lsum_codes, p_levels=255)
        if lsum_codes:
            lw = alpha * (94 + 255) / 255 + (255 + 94) / 255
        else:
            lw = alpha * (math.exp(-1) + 1) + (1 + math.exp(-1))
        assert l[0] == pytest.approx(lw, rel=1e-15)
        np.testing.assert_allclose(O[0], [0.5 * x / (255 * lw) for x in acc], rtol=1e-13)


def test_uint8_p_codes_use_the_full_byte():
    # one key block, logits spread over [-6, 0]: RNE(255 p) reaches 255 at the
    # row max and the code-weighted mean with the codes recomputed from the
    # logits by hand (t_j = a b_j sQ sK / sqrt(d) with S_0j = a b_j)
    d = 128
    a = 127
    b = list(range(-127, 1, 8))             # 16 keys
    L = len(b)
    Qq = np.zeros((L, d), np.int8)
    Qq[0, 0] = a
    Kq = np.zeros((L, d), np.int8)
    Kq[:, 0] = b
    sQ = np.full(L, 0.0625, np.float32)
    sK = np.full(L, 0.0625, np.float32)
    rng = np.random.default_rng(33)
    Vq = rand_i8(rng, L, d)
    t = [a * bj * 0.0625 * 0.0625 / math.sqrt(d) for bj in b]
    mx = max(t)
    codes = [round(255 * math.exp(tj - mx)) for tj in t]
    assert max(codes) == 255 and min(codes) < 127
    O = oracle.attention_online_rows(Qq, Kq, Vq, sQ, sK, 0.5, False, 128, r0=0, r1=1, lsum_codes=True,
                                     p_levels=255)
    want = [0.5 * sum(codes[j] * int(Vq[j, c]) for j in range(L)) / sum(codes) for c in range(d)]
    np.testing.assert_allclose(O[0], want, rtol=1e-13)


def test_uint8_p_rejects_other_levels():
    Qq = np.zeros((4, 64), np.int8)
    s = np.ones(4, np.float32)
    with pytest.raises(ValueError):
        oracle.attention_online_rows(Qq, Qq, Qq, s, s, 1.0, False, p_levels=128)


def test_uint8_p_error_below_int8_p():
    # IntAttention Table 5: UINT8 P (range [0, 1] over all 256 codes) keeps
    # attention closer to full precision than signed INT8 P (half the codes).
    # Same quantised Q / K / V, online form, against fp64 attention of the
    # unquantised inputs: cosine similarity higher and RMSE lower.
    rng = np.random.default_rng(34)
    L, d = 512, 64
    q, k, v = (rng.standard_normal((L, d)).astype(np.float32) for _ in range(3))
    Qq, sQ = oracle.quantize_per_token(q)
    Kq, sK = oracle.quantize_per_token(k)
    Vq, sV = oracle.quantize_per_tensor(v, 1)
    ref = oracle.attention_fp64_rows(q.astype(np.float64), k.astype(np.float64), v.astype(np.float64), True)
    stats = {}
    for lv in (127, 255):
        O = oracle.attention_online_rows(Qq, Kq, Vq, sQ, sK, float(sV[0]), True, 128, p_levels=lv)
        cos = (O * ref).sum() / math.sqrt((O * O).sum() * (ref * ref).sum())
        rmse = math.sqrt(((O - ref) ** 2).mean())
        stats[lv] = (cos, rmse)
    assert stats[255][0] > stats[127][0]
    assert stats[255][1] < stats[127][1]
