"""The attention kernel with Q quantised inside it (intfa_attention_fwd_q16)
against the path that quantises Q with intfa_quantize_per_token first: the
per-token codes and scales are the same arithmetic, so O and s_Q must agree
bit for bit; and the fused path against the oracle through intfa_forward."""
import numpy as np
import pytest
import torch

from int8_quantized_attention_token_b200 import intfa
from int8_quantized_attention_token_b200.workloads import make_qkv
from parity import TOL_MAXABS, TOL_MRE, gap, oracle_heads

pytestmark = pytest.mark.gpu


def both_paths(Q, K, V, causal):
    B, H, L, d = Q.shape
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    Qq, sQ = intfa.intfa_quantize_per_token(Qd)
    Kq, sK = intfa.intfa_quantize_per_token(Kd)
    Vt, sV = intfa.intfa_quantize_per_tensor(Vd.reshape(B * H, L, d), transpose=True)
    Vt, sV = Vt.reshape(B, H, d, -1), sV.reshape(B, H)
    O_ref = intfa.intfa_attention_fwd(Qq, Kq, Vt, sQ, sK, sV, causal)
    sQ_f = torch.full_like(sQ, float("nan"))
    O_f = intfa.intfa_attention_fwd_q16(Qd, Kq, Vt, sK, sV, causal, s_Q=sQ_f)
    O_n = intfa.intfa_attention_fwd_q16(Qd, Kq, Vt, sK, sV, causal)   # no s_Q output
    torch.cuda.synchronize()
    assert intfa.intfa_device_status(clear=True) == 0
    return O_ref, O_f, O_n, sQ, sQ_f


@pytest.mark.parametrize("B,H,L,d,causal", [
    (1, 1, 128, 64, False),
    (1, 2, 256, 128, True),
    (2, 3, 333, 64, True),           # ragged last query tile (rows past L are zero)
    (1, 2, 1000, 128, False),
    (1, 1, 1, 128, True),
    (2, 2, 640, 64, False),
    (1, 3, 2050, 128, True),         # 17 tiles per head: several tiles per CTA below
])
def test_fused_q_bit_identical(B, H, L, d, causal):
    Q, K, V = make_qkv(B, H, L, d, seed=3 * L + d + causal)
    O_ref, O_f, O_n, sQ, sQ_f = both_paths(Q, K, V, causal)
    assert torch.equal(O_f, O_ref)
    assert torch.equal(O_n, O_ref)
    assert torch.equal(sQ_f, sQ)


def test_fused_q_outlier_channels():
    """Q with outlier channels and tokens (per-token scales vary by 100x)."""
    Q, K, V = make_qkv(2, 2, 512, 128, seed=11)
    Q[:, :, :, 5] *= 20.0
    Q[0, 1, 7] *= 8.0
    O_ref, O_f, _, sQ, sQ_f = both_paths(Q, K, V, True)
    assert torch.equal(O_f, O_ref)
    assert torch.equal(sQ_f, sQ)


def test_fused_q_many_tiles_per_cta():
    """More query tiles than SMs, so each persistent CTA walks several tiles
    (and both Q buffers and the s_Q ring wrap)."""
    B, H, L, d = 4, 8, 4096, 128
    Q, K, V = make_qkv(B, H, L, d, seed=5)
    O_ref, O_f, _, sQ, sQ_f = both_paths(Q, K, V, True)
    assert torch.equal(O_f, O_ref)
    assert torch.equal(sQ_f, sQ)


@pytest.mark.parametrize("L,d,causal", [(700, 128, True), (384, 64, False)])
def test_forward_matches_oracle(L, d, causal):
    """intfa_forward (K, V quantisers + fused-Q attention) against the oracle."""
    Q, K, V = make_qkv(1, 2, L, d, seed=L)
    O = intfa.intfa_forward(Q.cuda(), K.cuda(), V.cuda(), causal).float().cpu().numpy()
    heads = [(0, 0), (0, 1)]
    ref = oracle_heads(Q, K, V, causal, heads)
    got = np.stack([O[b, h] for b, h in heads])
    want = np.stack([ref[k]["O"] for k in heads])
    mx, mre = gap(got, want)
    assert mx <= TOL_MAXABS and mre <= TOL_MRE, (mx, mre)
