"""Test forms of the fused attention kernel (intfa_debug_attention_scores,
intfa_debug_wait_timeout), through the C ABI.

* The integer logits S = Q_hat K_hat^T (IntAttention eq. 4) exactly as the
  kernel's softmax recovers them from its tensor-memory accumulator (an fp16
  MMA presets the accumulator to 1.5 * 2^23, the INT8 MMAs add their int32
  sums, the float read minus 1.5 * 2^23 is S): bit-exact against the
  oracle's int32 product, including the +-127^2 d extremes; key blocks the
  kernel never computes stay untouched; the output O is the release
  kernel's, bit for bit.
* A bounded wait running out: the kernel form that issues no copy and no
  MMA gives up on its first wait, records the site in the status word and
  returns; the device stays usable and the next call is correct.
"""
import numpy as np
import pytest
import torch

import oracle
from int8_quantized_attention_token_b200 import intfa
from int8_quantized_attention_token_b200.workloads import make_qkv
from parity import TOL_MAXABS, TOL_MRE, gap, oracle_heads

pytestmark = pytest.mark.gpu

SENTINEL = -(2 ** 31)


def random_codes(B, H, L, d, seed, extremes=False):
    g = torch.Generator().manual_seed(seed)
    Qq = torch.randint(-127, 128, (B, H, L, d), generator=g, dtype=torch.int8)
    Kq = torch.randint(-127, 128, (B, H, L, d), generator=g, dtype=torch.int8)
    if extremes:
        Qq[..., 0, :] = 127
        Kq[..., 0, :] = 127
        if L > 1:
            Kq[..., 1, :] = -127
    ld = intfa.intfa_vt_ld(L)
    Vt = torch.randint(-127, 128, (B, H, d, ld), generator=g, dtype=torch.int8)
    # small positive scales: the softmax stays well-conditioned even at 127^2 d
    sQ = torch.rand(B, H, L, generator=g) * 1e-3 + 1e-4
    sK = torch.rand(B, H, L, generator=g) * 1e-3 + 1e-4
    sV = torch.rand(B, H, generator=g) + 0.5
    return Qq, Kq, Vt, sQ, sK, sV


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("B,H,L,causal", [(1, 1, 1, False), (1, 1, 45, True), (1, 2, 200, False),
                                          (2, 1, 384, True), (1, 1, 640, True), (1, 3, 300, False)])
def test_scores_from_the_production_accumulator(B, H, L, d, causal):
    args = random_codes(B, H, L, d, seed=L * 7 + d + causal, extremes=(L == 200))
    dev = [a.cuda() for a in args]
    S = torch.full((B, H, L, L), SENTINEL, dtype=torch.int32, device="cuda")
    O = intfa.intfa_debug_attention_scores(*dev, causal, S)
    O_rel = intfa.intfa_attention_fwd(*dev, causal)
    torch.cuda.synchronize()
    assert intfa.intfa_device_status(clear=True) == 0
    assert torch.equal(O, O_rel)      # the debug form changes nothing else
    Qq, Kq = args[0], args[1]
    So = oracle.qk_int32(Qq.reshape(B * H, L, d).numpy(), Kq.reshape(B * H, L, d).numpy()).reshape(B, H, L, L)
    got = S.cpu().numpy()
    q = np.arange(L)[:, None]
    k = np.arange(L)[None, :]
    # key blocks the kernel computes: all, or (causal) up to the query tile's diagonal block
    done = np.ones((L, L), bool) if not causal else (k // 128) <= (q // 128)
    np.testing.assert_array_equal(got[..., done], So[..., done])
    assert (got[..., ~done] == SENTINEL).all()
    if L == 200:
        assert So[0, 0, 0, 0] == 127 * 127 * d and So[0, 0, 0, 1] == -127 * 127 * d
        assert got[0, 0, 0, 0] == 127 * 127 * d and got[0, 0, 0, 1] == -127 * 127 * d


def test_bounded_wait_runs_out_and_the_device_stays_usable():
    torch.cuda.set_device(0)
    B, H, L, d = 1, 2, 256, 64
    Q, K, V = make_qkv(B, H, L, d, seed=31)
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    Qq, sQ = intfa.intfa_quantize_per_token(Qd)
    Kq, sK = intfa.intfa_quantize_per_token(Kd)
    Vt, sV = intfa.intfa_quantize_per_tensor(Vd.reshape(B * H, L, d), transpose=True)
    args = (Qq, Kq, Vt.reshape(B, H, d, -1), sQ, sK, sV.reshape(B, H))
    torch.cuda.synchronize()
    assert intfa.intfa_device_status(clear=True) == 0
    O = torch.zeros(B, H, L, d, dtype=torch.float16, device="cuda")
    intfa.intfa_debug_wait_timeout(*args, True, 20000, O=O)
    torch.cuda.synchronize()
    w = intfa.intfa_device_status(clear=True)
    # 0x100 | site of the first wait to run out: the tensor-core issuer's wait
    # for its Q tile (2), the output warps' wait for a P V block (9), or the
    # softmax's wait for S (12)
    assert w & 0x100 and (w & 0xFF) in (2, 9, 12), hex(w)
    assert not O.any()                         # nothing was written
    assert intfa.intfa_device_status(clear=True) == 0
    # the device is still usable: a normal call afterwards matches the oracle
    O = intfa.intfa_attention_fwd(*args, True)
    torch.cuda.synchronize()
    assert intfa.intfa_device_status(clear=True) == 0
    ref = oracle_heads(Q, K, V, True, [(0, 0), (0, 1)])
    for h in range(H):
        mx, mre = gap(O[0, h].float().cpu().numpy(), ref[(0, h)]["O"])
        assert mx <= TOL_MAXABS and mre <= TOL_MRE, (mx, mre)
