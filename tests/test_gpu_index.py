"""The IndexSoftmax attention kernel (IntAttention sections 3.1-3.2) against
the oracle: the integer row max of Q_hat K_hat^T and the integer row sum of
the UINT8 table values bit for bit, O within fp16 rounding.  Both sides
quantise the same seeded fp16 inputs per tensor, each with its own quantiser
(bit-identical by the quantiser parity tests)."""
import numpy as np
import pytest
import torch

import oracle
from int8_quantized_attention_token_b200 import intfa
from int8_quantized_attention_token_b200.workloads import make_qkv

pytestmark = pytest.mark.gpu

# fp16 output against the fp64 oracle: one rounding to fp16 (<= 2^-11 of the
# value) plus fp32 arithmetic in the epilogue
TOL_MAXABS = 1e-3


def run_gpu(Q, K, V, causal, c, b):
    B, H, L, d = Q.shape
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    Qq, sQ = intfa.intfa_quantize_per_tensor(Qd.reshape(B * H, L, d), transpose=False)
    Kq, sK = intfa.intfa_quantize_per_tensor(Kd.reshape(B * H, L, d), transpose=False)
    Vt, sV = intfa.intfa_quantize_per_tensor(Vd.reshape(B * H, L, d), transpose=True)
    m = torch.full((B, H, L), -7, dtype=torch.int32, device="cuda")
    l = torch.full((B, H, L), -7, dtype=torch.int32, device="cuda")
    O = intfa.intfa_index_attention_fwd(Qq.reshape(B, H, L, d), Kq.reshape(B, H, L, d),
                                        Vt.reshape(B, H, d, -1), sQ.reshape(B, H), sK.reshape(B, H),
                                        sV.reshape(B, H), causal, c, b, m_out=m, l_out=l)
    torch.cuda.synchronize()
    assert intfa.intfa_device_status(clear=True) == 0
    return O.float().cpu().numpy(), m.cpu().numpy(), l.cpu().numpy()


def oracle_head(Q, K, V, bb, h, causal, c, b, r0=0, r1=None):
    q, k, v = (X[bb, h].float().numpy() for X in (Q, K, V))
    Qq, sQ = oracle.quantize_per_tensor(q, 1)
    Kq, sK = oracle.quantize_per_tensor(k, 1)
    Vq, sV = oracle.quantize_per_tensor(v, 1)
    return oracle.index_attention_rows(Qq, Kq, Vq, float(sQ[0]), float(sK[0]), float(sV[0]), causal,
                                       c, b, r0, r1, want_stats=True)


def check(Q, K, V, causal, c=6.6, b=5):
    B, H, L, d = Q.shape
    O, m, l = run_gpu(Q, K, V, causal, c, b)
    assert np.isfinite(O).all()
    for bb in range(B):
        for h in range(H):
            Oo, mo, lo = oracle_head(Q, K, V, bb, h, causal, c, b)
            np.testing.assert_array_equal(m[bb, h], mo)
            np.testing.assert_array_equal(l[bb, h], lo)
            scale = np.abs(Oo).max()
            assert np.abs(O[bb, h] - Oo).max() <= TOL_MAXABS * scale


@pytest.mark.parametrize("B,H,L,d,causal", [
    (1, 2, 300, 64, False),      # ragged last block, 3 key blocks
    (2, 3, 777, 128, True),      # ragged causal, 7 tiles
    (1, 1, 128, 128, False),     # exactly one block
    (1, 2, 1000, 128, True),
    (1, 1, 1, 64, False),        # a single key
    (1, 1, 129, 128, True),      # one full tile and a one-row tail
])
def test_index_attention_matches_oracle(B, H, L, d, causal):
    Q, K, V = make_qkv(B, H, L, d, seed=100 + L + d)
    check(Q, K, V, causal)


@pytest.mark.parametrize("c,b", [(6.6, 8), (4.0, 3), (12.0, 5), (6.6, 1)])
def test_index_attention_table_parameters(c, b):
    # b = 8 with N(0, 1) inputs puts c_int above 2^15: the integer-quotient path
    Q, K, V = make_qkv(1, 2, 640, 128, seed=7)
    check(Q, K, V, True, c, b)


def test_index_attention_tiny_scales_take_the_integer_path():
    # inputs of magnitude ~1e-3: c_int far above 2^18, idx by integer division
    Q, K, V = make_qkv(1, 1, 384, 64, seed=8)
    Q, K = (Q.float() * 1e-3).half(), (K.float() * 1e-3).half()
    check(Q, K, V, False)


def test_index_attention_constant_logits():
    # Q = 0: every table value is 255 and O is s_V times the mean of V_hat
    Q, K, V = make_qkv(1, 2, 256, 128, seed=9)
    Q = torch.zeros_like(Q)
    check(Q, K, V, True)


def test_index_attention_full_size_sampled_rows():
    # the benchmark's shape: B = 4, H = 32, L = 4096, d = 128, causal; the
    # oracle checks sampled rows of sampled heads
    B, H, L, d = 4, 32, 4096, 128
    Q, K, V = make_qkv(B, H, L, d, seed=0)
    O, m, l = run_gpu(Q, K, V, True, 6.6, 5)
    rng = np.random.default_rng(1)
    for (bb, h) in [(0, 0), (3, 31), (1, 17)]:
        for r0 in [0, int(rng.integers(1, L - 8)), L - 8]:
            Oo, mo, lo = oracle_head(Q, K, V, bb, h, True, 6.6, 5, r0, r0 + 8)
            np.testing.assert_array_equal(m[bb, h, r0:r0 + 8], mo)
            np.testing.assert_array_equal(l[bb, h, r0:r0 + 8], lo)
            assert np.abs(O[bb, h, r0:r0 + 8] - Oo).max() <= TOL_MAXABS * np.abs(Oo).max()
