"""The fused kernel with the row sum taken from the P codes (the other
reading of the pages' row sum) against the oracle's online form with the same
reading, on the benchmark's kind of inputs."""
import numpy as np
import pytest
import torch

import oracle
from int8_quantized_attention_token_b200 import intfa
from int8_quantized_attention_token_b200.workloads import make_qkv
from parity import TOL_MAXABS, TOL_MRE, gap

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,L,d,causal,outliers", [
    (1, 2, 777, 128, True, False),
    (1, 2, 1000, 64, False, True),
    (2, 1, 256, 128, False, False),
])
def test_codesum_matches_oracle(B, H, L, d, causal, outliers):
    Q, K, V = make_qkv(B, H, L, d, seed=400 + L, outliers=outliers)
    Qq, sQ = intfa.intfa_quantize_per_token(Q.cuda())
    Kq, sK = intfa.intfa_quantize_per_token(K.cuda())
    Vt, sV = intfa.intfa_quantize_per_tensor(V.cuda().reshape(B * H, L, d), transpose=True)
    O = intfa.intfa_attention_fwd_codesum(Qq, Kq, Vt.reshape(B, H, d, -1), sQ, sK, sV.reshape(B, H), causal)
    torch.cuda.synchronize()
    assert intfa.intfa_device_status(clear=True) == 0
    O = O.float().cpu().numpy()
    got, want = [], []
    for b in range(B):
        for h in range(H):
            q, k, v = (X[b, h].float().numpy() for X in (Q, K, V))
            qq, sq = oracle.quantize_per_token(q)
            kq, sk = oracle.quantize_per_token(k)
            vq, sv = oracle.quantize_per_tensor(v, 1)
            want.append(oracle.attention_online_rows(qq, kq, vq, sq, sk, float(sv[0]), causal, 128,
                                                     lsum_codes=True))
            got.append(O[b, h])
    mx, mre = gap(np.stack(got), np.stack(want))
    assert mx <= TOL_MAXABS and mre <= TOL_MRE, (mx, mre)
