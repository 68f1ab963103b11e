"""b-bit (INT4) per-token Q / K codes: the GPU quantiser bit-exact against
the oracle's (codes and scale bit patterns), b = 8 identical to the INT8
quantiser, and the fused attention on 4-bit codes against the oracle's online
form on the same codes; its error against fp64 attention is reported."""
import numpy as np
import pytest
import torch

import oracle
from int8_quantized_attention_token_b200 import intfa
from int8_quantized_attention_token_b200.workloads import make_qkv
from parity import TOL_MAXABS, TOL_MRE, gap

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bits,d", [(4, 128), (4, 64), (3, 256), (6, 8), (2, 32)])
def test_bits_quantiser_bit_exact(bits, d):
    g = torch.Generator().manual_seed(bits * 1000 + d)
    x = (torch.randn(777, d, generator=g) * 3).half()
    x[5] = 0                                                  # an all-zero row
    x[6, :4] = torch.tensor([1.75, 0.5, 0.625, 0.875])      # ties when 4-bit
    x[6, 4:] = 0
    q, s = intfa.intfa_quantize_per_token_bits(x.cuda(), bits)
    torch.cuda.synchronize()
    oq, os_ = oracle.quantize_per_token_bits(x.float().numpy(), bits)
    np.testing.assert_array_equal(q.cpu().numpy(), oq)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), os_.view(np.uint32))


def test_bits8_equals_int8_quantiser():
    g = torch.Generator().manual_seed(1)
    x = (torch.randn(1000, 128, generator=g) * 2).half().cuda()
    q8, s8 = intfa.intfa_quantize_per_token(x)
    qb, sb = intfa.intfa_quantize_per_token_bits(x, 8)
    torch.cuda.synchronize()
    assert torch.equal(q8, qb) and torch.equal(s8.view(torch.int32), sb.view(torch.int32))


@pytest.mark.parametrize("causal", [False, True])
def test_attention_on_int4_codes(causal):
    B, H, L, d = 1, 2, 640, 128
    Q, K, V = make_qkv(B, H, L, d, seed=600 + causal)
    Qq, sQ = intfa.intfa_quantize_per_token_bits(Q.cuda(), 4)
    Kq, sK = intfa.intfa_quantize_per_token_bits(K.cuda(), 4)
    Vt, sV = intfa.intfa_quantize_per_tensor(V.cuda().reshape(B * H, L, d), transpose=True)
    O = intfa.intfa_attention_fwd(Qq, Kq, Vt.reshape(B, H, d, -1), sQ, sK, sV.reshape(B, H), causal)
    torch.cuda.synchronize()
    assert intfa.intfa_device_status(clear=True) == 0
    O = O.float().cpu().numpy()
    got, want, ref64 = [], [], []
    for h in range(H):
        q, k, v = (X[0, h].float().numpy() for X in (Q, K, V))
        qq, sq = oracle.quantize_per_token_bits(q, 4)
        kq, sk = oracle.quantize_per_token_bits(k, 4)
        vq, sv = oracle.quantize_per_tensor(v, 1)
        want.append(oracle.attention_online_rows(qq, kq, vq, sq, sk, float(sv[0]), causal, 128))
        ref64.append(oracle.attention_fp64_rows(q, k, v, causal))
        got.append(O[0, h])
    got, want, ref64 = np.stack(got), np.stack(want), np.stack(ref64)
    mx, mre = gap(got, want)
    assert mx <= TOL_MAXABS and mre <= TOL_MRE, (mx, mre)
    print(f"\nINT4 Q/K, causal={causal}: error against fp64 GPU {gap(got, ref64)}, oracle {gap(want, ref64)}")
