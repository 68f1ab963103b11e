"""The tensor-core (tcgen05 kind::i8) Q_hat K_hat^T against the oracle's
exact int32 product, bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from int8_quantized_attention_token_b200 import intfa

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("B,H,L", [(1, 1, 128), (1, 2, 200), (2, 1, 384), (1, 1, 1), (1, 1, 45)])
def test_qk_bit_exact(B, H, L, d):
    g = torch.Generator().manual_seed(B * 100 + H * 10 + L + d)
    Qq = torch.randint(-127, 128, (B, H, L, d), generator=g, dtype=torch.int8)
    Kq = torch.randint(-127, 128, (B, H, L, d), generator=g, dtype=torch.int8)
    S = intfa.intfa_debug_qk(Qq.cuda(), Kq.cuda()).cpu().numpy()
    So = oracle.qk_int32(Qq.reshape(B * H, L, d).numpy(), Kq.reshape(B * H, L, d).numpy())
    np.testing.assert_array_equal(S.reshape(B * H, L, L), So)


@pytest.mark.parametrize("d", [64, 128])
def test_qk_extremes(d):
    L = 256
    Qq = torch.full((1, 1, L, d), 127, dtype=torch.int8)
    Kq = torch.full((1, 1, L, d), 127, dtype=torch.int8)
    Kq[0, 0, 1::2] = -127
    Qq[0, 0, 3] = -127
    S = intfa.intfa_debug_qk(Qq.cuda(), Kq.cuda()).cpu().numpy()[0, 0]
    So = oracle.qk_int32(Qq[0].numpy(), Kq[0].numpy())[0]
    np.testing.assert_array_equal(S, So)
    assert S[0, 0] == 127 * 127 * d and S[0, 1] == -127 * 127 * d
