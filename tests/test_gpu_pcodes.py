"""P codes over the full byte: the fused kernel with P_hat = RNE(255 p) stored
as UINT8 and multiplied as unsigned tensor-core operands (the unsigned scheme
of IntAttention's Table 5 ablation) against the oracle's online form with the
same code range, through intfa_attention_fwd_pcodes; the entry's 127-level
settings against the INT8 entry points bit for bit; and the Table 5 ordering
(UINT8 P closer to unquantised attention than INT8 P) on the kernel's own
outputs."""
import math

import numpy as np
import pytest
import torch

from int8_quantized_attention_token_b200 import intfa
from int8_quantized_attention_token_b200.workloads import by_name, make_qkv, make_workload
from parity import TOL_MAXABS, TOL_MRE, gap, oracle_heads

pytestmark = pytest.mark.gpu


def quantise(Q, K, V):
    B, H, L, d = Q.shape
    Qq, sQ = intfa.intfa_quantize_per_token(Q.cuda())
    Kq, sK = intfa.intfa_quantize_per_token(K.cuda())
    Vt, sV = intfa.intfa_quantize_per_tensor(V.cuda().reshape(B * H, L, d), transpose=True)
    return Qq, Kq, Vt.reshape(B, H, d, -1), sQ, sK, sV.reshape(B, H)


def run(args, causal, p_levels, lsum_codes):
    O = intfa.intfa_attention_fwd_pcodes(*args, causal, p_levels=p_levels, lsum_codes=lsum_codes)
    torch.cuda.synchronize()
    assert intfa.intfa_device_status(clear=True) == 0
    return O


@pytest.mark.parametrize("B,H,L,d,causal,outliers", [
    (1, 2, 777, 128, True, False),     # ragged causal, 7 tiles
    (1, 2, 1000, 64, False, True),     # ragged, d = 64, outlier channels / tokens
    (2, 1, 256, 128, False, False),
    (1, 1, 1, 64, False, False),       # a single key
    (1, 1, 129, 128, True, False),     # one full tile and a one-row tail
])
@pytest.mark.parametrize("lsum_codes", [False, True])
def test_uint8_p_matches_oracle(B, H, L, d, causal, outliers, lsum_codes):
    Q, K, V = make_qkv(B, H, L, d, seed=500 + L + d, outliers=outliers)
    O = run(quantise(Q, K, V), causal, 255, lsum_codes).float().cpu().numpy()
    heads = [(b, h) for b in range(B) for h in range(H)]
    ref = oracle_heads(Q, K, V, causal, heads, p_levels=255, lsum_codes=lsum_codes)
    got = np.stack([O[b, h] for b, h in heads])
    want = np.stack([ref[k]["O"] for k in heads])
    assert np.isfinite(got).all()
    mx, mre = gap(got, want)
    assert mx <= TOL_MAXABS and mre <= TOL_MRE, (mx, mre)


@pytest.mark.parametrize("d", [64, 128])
def test_127_levels_equal_the_int8_entry_points(d):
    B, H, L = 1, 2, 640
    Q, K, V = make_qkv(B, H, L, d, seed=600 + d)
    args = quantise(Q, K, V)
    O0 = intfa.intfa_attention_fwd(*args, True)
    O1 = intfa.intfa_attention_fwd_codesum(*args, True)
    P0 = run(args, True, 127, False)
    P1 = run(args, True, 127, True)
    assert torch.equal(O0.view(torch.int16), P0.view(torch.int16))
    assert torch.equal(O1.view(torch.int16), P1.view(torch.int16))


def test_uint8_p_constant_logits():
    # Q = 0: every code is 255 and O is s_V times the mean of the visible V_hat
    B, H, L, d = 1, 2, 300, 128
    Q, K, V = make_qkv(B, H, L, d, seed=601)
    Q = torch.zeros_like(Q)
    args = quantise(Q, K, V)
    O = run(args, True, 255, False).float().cpu().numpy()
    Vt, sV = args[2].cpu(), args[5].cpu()
    for h in range(H):
        v = Vt[0, h, :, :L].T.double().numpy()
        want = float(sV[0, h]) * np.cumsum(v, axis=0) / np.arange(1, L + 1)[:, None]
        np.testing.assert_allclose(O[0, h], want, rtol=0, atol=1e-3 * np.abs(want).max())


def test_uint8_p_full_size_sampled_rows():
    # the benchmark's shape (B = 4, H = 32, L = 4096, d = 128, causal), sampled
    # rows of sampled heads against the oracle
    w = by_name("attn_B4_H32_L4096_d128_causal")
    Q, K, V = make_workload(w)
    O = run(quantise(Q, K, V), True, 255, False).float().cpu().numpy()
    rng = np.random.default_rng(2)
    rows = np.unique(np.concatenate([np.arange(0, 4), np.arange(w.L - 4, w.L),
                                     rng.choice(w.L, 24, replace=False)]))
    heads = [(0, 0), (3, 31), (2, 9)]
    ref = oracle_heads(Q, K, V, True, heads, rows=rows, p_levels=255)
    got = np.stack([O[b, h][rows] for b, h in heads])
    want = np.stack([ref[k]["O"] for k in heads])
    mx, mre = gap(got, want)
    assert mx <= TOL_MAXABS and mre <= TOL_MRE, (mx, mre)


def test_uint8_p_closer_to_fp64_than_int8_p():
    # IntAttention Table 5 on the kernel's outputs: cosine similarity to
    # unquantised fp64 attention higher and RMSE lower with UINT8 P
    B, H, L, d = 1, 4, 1024, 128
    Q, K, V = make_qkv(B, H, L, d, seed=602)
    args = quantise(Q, K, V)
    heads = [(0, h) for h in range(H)]
    ref = oracle_heads(Q, K, V, True, heads, fp64=True)
    x = np.stack([ref[k]["Ox"] for k in heads])
    stats = {}
    for lv in (127, 255):
        O = run(args, True, lv, False).double().cpu().numpy()[0]
        cos = float((O * x).sum() / math.sqrt((O * O).sum() * (x * x).sum()))
        rmse = float(np.sqrt(((O - x) ** 2).mean()))
        stats[lv] = (cos, rmse)
    print(f"\nINT8 P: cosine {stats[127][0]:.6f} RMSE {stats[127][1]:.3e}; "
          f"UINT8 P: cosine {stats[255][0]:.6f} RMSE {stats[255][1]:.3e}")
    assert stats[255][0] > stats[127][0]
    assert stats[255][1] < stats[127][1]
