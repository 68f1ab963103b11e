"""Group-wise (per-block) Q / K scales (IntAttention section 3.3): the fused
kernel with one scale per block of tokens against the oracle's block-wise
online form given the same per-block quantisation, and bit-identity with the
per-token entry point when the per-block scales are written out per token."""
import numpy as np
import pytest
import torch

import oracle
from int8_quantized_attention_token_b200 import intfa
from int8_quantized_attention_token_b200.workloads import make_qkv
from parity import TOL_MAXABS, TOL_MRE, gap

pytestmark = pytest.mark.gpu


def quantize_blocks_gpu(X, blk):
    B, H, L, d = X.shape
    q, s = intfa.intfa_quantize_per_tensor(X.cuda().reshape(B * H * L // blk, blk, d), transpose=False)
    return q.reshape(B, H, L, d), s.reshape(B, H, L // blk)


def run_gpu(Q, K, V, causal, blk):
    B, H, L, d = Q.shape
    Qq, sQ = quantize_blocks_gpu(Q, blk)
    Kq, sK = quantize_blocks_gpu(K, blk)
    Vt, sV = intfa.intfa_quantize_per_tensor(V.cuda().reshape(B * H, L, d), transpose=True)
    Vt, sV = Vt.reshape(B, H, d, -1), sV.reshape(B, H)
    O = intfa.intfa_attention_fwd_blockscale(Qq, Kq, Vt, sQ, sK, sV, causal, blk)
    torch.cuda.synchronize()
    assert intfa.intfa_device_status(clear=True) == 0
    return O, (Qq, Kq, Vt, sQ, sK, sV)


def oracle_head(Q, K, V, b, h, causal, blk):
    q, k, v = (X[b, h].float().numpy() for X in (Q, K, V))
    L, d = q.shape
    Qq, sQ = oracle.quantize_per_tensor(q.reshape(L // blk, blk * d), L // blk)
    Kq, sK = oracle.quantize_per_tensor(k.reshape(L // blk, blk * d), L // blk)
    Vq, sV = oracle.quantize_per_tensor(v, 1)
    return oracle.attention_online_rows(Qq.reshape(L, d), Kq.reshape(L, d), Vq, np.repeat(sQ, blk),
                                        np.repeat(sK, blk), float(sV[0]), causal, 128)


@pytest.mark.parametrize("B,H,L,d,causal,blk", [
    (1, 2, 512, 128, True, 128),
    (1, 2, 384, 64, False, 64),
    (2, 1, 256, 128, True, 16),
    (1, 1, 768, 128, False, 256),
    (1, 1, 256, 64, True, 1),
])
def test_blockscale_matches_oracle(B, H, L, d, causal, blk):
    Q, K, V = make_qkv(B, H, L, d, seed=200 + blk + L, outliers=True)
    O, _ = run_gpu(Q, K, V, causal, blk)
    O = O.float().cpu().numpy()
    got = np.stack([O[b, h] for b in range(B) for h in range(H)])
    want = np.stack([oracle_head(Q, K, V, b, h, causal, blk) for b in range(B) for h in range(H)])
    mx, mre = gap(got, want)
    assert np.isfinite(got).all()
    assert mx <= TOL_MAXABS and mre <= TOL_MRE, (mx, mre)


@pytest.mark.parametrize("blk", [32, 128])
def test_blockscale_equals_per_token_entry_with_expanded_scales(blk):
    B, H, L, d = 1, 2, 1024, 128
    Q, K, V = make_qkv(B, H, L, d, seed=300 + blk)
    O, (Qq, Kq, Vt, sQ, sK, sV) = run_gpu(Q, K, V, True, blk)
    O2 = intfa.intfa_attention_fwd(Qq, Kq, Vt, sQ.repeat_interleave(blk, dim=2).contiguous(),
                                   sK.repeat_interleave(blk, dim=2).contiguous(), sV, True)
    torch.cuda.synchronize()
    assert torch.equal(O.view(torch.int16), O2.view(torch.int16))
