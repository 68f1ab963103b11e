"""The oracle against its stored tiny case, and the seeded input generator."""
import json
import os

import numpy as np
import torch

import oracle
from int8_quantized_attention_token_b200.workloads import WORKLOADS, make_qkv

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "oracle_tiny.json")


def test_oracle_reproduces_golden_tiny_case():
    with open(GOLDEN) as f:
        g = json.load(f)
    c = g["case"]
    Q, K, V = (t.float().numpy().reshape(2, 8, 64)
               for t in make_qkv(c["B"], c["H"], c["L"], c["d"], seed=c["seed"]))
    Qq, sQ = oracle.quantize_per_token(Q)
    Kq, sK = oracle.quantize_per_token(K)
    Vq, sV = oracle.quantize_per_tensor(V, 2)
    assert sQ.ravel().tolist() == np.array(g["sQ"], np.float32).ravel().tolist()
    assert sK.ravel().tolist() == np.array(g["sK"], np.float32).ravel().tolist()
    assert sV.tolist() == np.array(g["sV"], np.float32).tolist()
    assert int(Qq.astype(np.int64).sum()) == g["Qq_sum"]
    assert int(Vq.astype(np.int64).sum()) == g["Vq_sum"]
    for causal, key in ((False, "O"), (True, "O_causal")):
        O = oracle.attention_fwd(Qq, Kq, Vq, sQ, sK, sV, causal)
        np.testing.assert_array_equal(O.ravel(), np.array(g[key]))


def test_generator_is_deterministic_and_shaped():
    a = make_qkv(1, 2, 40, 64, seed=5)
    b = make_qkv(1, 2, 40, 64, seed=5)
    c = make_qkv(1, 2, 40, 64, seed=6)
    for x, y in zip(a, b):
        assert x.dtype == torch.float16 and x.shape == (1, 2, 40, 64)
        assert torch.equal(x, y)
    assert not torch.equal(a[0], c[0])


def test_outlier_structure():
    Q, K, V = make_qkv(2, 4, 2000, 128, seed=0, outliers=True)
    Qf, Kf = Q.float(), K.float()
    ch_std = Qf.std(dim=(0, 1, 2))
    big = torch.nonzero(ch_std > 5).ravel()
    assert big.numel() == 1                                   # round(0.01 * 128) = 1 channel x20
    assert torch.equal(big, torch.nonzero(Kf.std(dim=(0, 1, 2)) > 5).ravel())
    base = Qf[..., [c for c in range(128) if c != int(big)]]
    tok_std = base.std(dim=(1, 3))                            # [B, L]
    for b in range(2):
        assert int((tok_std[b] > 4).sum()) == 2               # round(0.001 * 2000) = 2 tokens x8
    assert float(V.float().std()) < 1.1


def test_workload_table():
    assert [w.L for w in WORKLOADS] == [128, 1024, 4096, 4096, 16384]
    w = WORKLOADS[2]
    assert w.ops == 4 * 4 * 32 * 4096 * 4096 * 128 / 2
