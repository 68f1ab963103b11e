"""Decode (one query per head against an INT8 key / value cache, split-KV)
against the oracle's decode with the same key ranges.  Both sides quantise
the same seeded fp16 inputs with their own quantisers."""
import numpy as np
import pytest
import torch

import oracle
from int8_quantized_attention_token_b200 import intfa
from parity import TOL_MAXABS, TOL_MRE, gap

pytestmark = pytest.mark.gpu


def make(B, H, L, d, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    q = (torch.randn(B, H, d, generator=g) * scale).half()
    K = (torch.randn(B, H, L, d, generator=g) * scale).half()
    V = torch.randn(B, H, L, d, generator=g).half()
    return q, K, V


def run_gpu(q, K, V, splits):
    B, H, L, d = K.shape
    Kq, sK = intfa.intfa_quantize_per_token(K.cuda())
    Vq, sV = intfa.intfa_quantize_per_tensor(V.cuda().reshape(B * H, L, d), transpose=False)
    O = intfa.intfa_decode_fwd(q.cuda(), Kq, sK, Vq.reshape(B, H, L, d), sV.reshape(B, H), splits)
    torch.cuda.synchronize()
    assert intfa.intfa_device_status(clear=True) == 0
    return O.float().cpu().numpy()


def oracle_decode(q, K, V, b, h, splits):
    L, d = K.shape[2], K.shape[3]
    qq, sq = oracle.quantize_per_token(q[b, h].float().numpy()[None, :])
    Kq, sK = oracle.quantize_per_token(K[b, h].float().numpy())
    Vq, sV = oracle.quantize_per_tensor(V[b, h].float().numpy(), 1)
    nblk = -(-L // 128)
    split_len = -(-nblk // splits) * 128
    return oracle.decode(qq[0], float(sq[0]), Kq, sK, Vq, float(sV[0]), 128, split_len)


@pytest.mark.parametrize("B,H,L,d,splits", [
    (1, 2, 1000, 128, 1),
    (2, 3, 4097, 64, 3),      # ragged last block, uneven ranges
    (1, 1, 1, 128, 1),        # a single cache entry
    (1, 2, 300, 128, 8),      # more ranges than blocks: empty ranges
    (2, 2, 8192, 128, 4),
    (1, 4, 2048, 64, 16),
])
def test_decode_matches_oracle(B, H, L, d, splits):
    q, K, V = make(B, H, L, d, seed=L + d + splits)
    O = run_gpu(q, K, V, splits)
    want = np.stack([oracle_decode(q, K, V, b, h, splits) for b in range(B) for h in range(H)])
    got = O.reshape(B * H, d)
    mx, mre = gap(got, want)
    assert np.isfinite(got).all()
    assert mx <= TOL_MAXABS and mre <= TOL_MRE, (mx, mre)


def test_decode_zero_query_is_mean_of_values():
    B, H, L, d = 1, 2, 700, 128
    q, K, V = make(B, H, L, d, seed=3)
    q = torch.zeros_like(q)
    O = run_gpu(q, K, V, 4)
    for h in range(H):
        Vq, sV = oracle.quantize_per_tensor(V[0, h].float().numpy(), 1)
        want = float(sV[0]) * Vq.astype(np.float64).mean(axis=0)
        assert np.abs(O[0, h] - want).max() <= 2e-3 * np.abs(want).max() + 1e-3
