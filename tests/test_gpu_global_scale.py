"""One V scale for the whole tensor (the per-tensor quantiser of IntAttention
eq. 3 applied to all heads together): codes and scale bit-exact against the
oracle's quantiser with one group, and the fused attention with that scale
against the oracle's online form."""
import numpy as np
import pytest
import torch

import oracle
from int8_quantized_attention_token_b200 import intfa
from int8_quantized_attention_token_b200.workloads import make_qkv
from parity import TOL_MAXABS, TOL_MRE, gap

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("transpose", [False, True])
def test_global_codes_and_scale_bit_exact(transpose):
    B, H, L, d = 2, 3, 300, 64
    _, _, V = make_qkv(B, H, L, d, seed=500, outliers=True)
    Vq, sV = intfa.intfa_quantize_global(V.cuda().reshape(B * H, L, d), transpose=transpose)
    torch.cuda.synchronize()
    Vq, sV = Vq.cpu().numpy(), sV.cpu().numpy()
    oq, os_ = oracle.quantize_per_tensor(V.float().numpy().reshape(B * H, L, d), 1)
    assert np.all(sV == os_[0])
    if transpose:
        ld = intfa.intfa_vt_ld(L)
        want = np.zeros((B * H, d, ld), np.int8)
        want[:, :, :L] = oq.transpose(0, 2, 1)
        np.testing.assert_array_equal(Vq, want)
    else:
        np.testing.assert_array_equal(Vq, oq)


def test_attention_with_global_value_scale():
    B, H, L, d = 1, 4, 640, 128
    Q, K, V = make_qkv(B, H, L, d, seed=501)
    Qq, sQ = intfa.intfa_quantize_per_token(Q.cuda())
    Kq, sK = intfa.intfa_quantize_per_token(K.cuda())
    Vt, sV = intfa.intfa_quantize_global(V.cuda().reshape(B * H, L, d), transpose=True)
    O = intfa.intfa_attention_fwd(Qq, Kq, Vt.reshape(B, H, d, -1), sQ, sK, sV.reshape(B, H), True)
    torch.cuda.synchronize()
    assert intfa.intfa_device_status(clear=True) == 0
    O = O.float().cpu().numpy()
    vq_all, sv_all = oracle.quantize_per_tensor(V.float().numpy().reshape(B * H, L, d), 1)
    got, want = [], []
    for h in range(H):
        q, k = Q[0, h].float().numpy(), K[0, h].float().numpy()
        qq, sq = oracle.quantize_per_token(q)
        kq, sk = oracle.quantize_per_token(k)
        want.append(oracle.attention_online_rows(qq, kq, vq_all[h], sq, sk, float(sv_all[0]), True, 128))
        got.append(O[0, h])
    mx, mre = gap(np.stack(got), np.stack(want))
    assert mx <= TOL_MAXABS and mre <= TOL_MRE, (mx, mre)
