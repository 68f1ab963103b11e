"""Quantisation error of the fused kernel and of the oracle against
unquantised fp64 attention (IntAttention eq. 1) on the five workloads, the
comparison INT-FlashAttention's abstract makes.  Sampled rows for the large
workloads.  The kernel must not be less accurate than the method it computes:
its error against fp64 stays within 10% (plus a small absolute margin) of the
oracle's.  Run with -s to see the table."""
import numpy as np
import pytest
import torch

from int8_quantized_attention_token_b200 import intfa
from int8_quantized_attention_token_b200.workloads import WORKLOADS, make_workload
from parity import gap, oracle_heads

pytestmark = pytest.mark.gpu


def run_gpu(Q, K, V, causal):
    B, H, L, d = Q.shape
    O = intfa.intfa_forward(Q.cuda(), K.cuda(), V.cuda(), causal)
    torch.cuda.synchronize()
    assert intfa.intfa_device_status(clear=True) == 0
    return O.float().cpu().numpy()


@pytest.mark.parametrize("w", WORKLOADS, ids=lambda w: w.name)
def test_error_against_fp64(w):
    Q, K, V = make_workload(w)
    O = run_gpu(Q, K, V, w.causal)
    rng = np.random.default_rng(0)
    if w.B * w.H * w.L <= 16 * 1024:
        heads = [(b, h) for b in range(w.B) for h in range(w.H)]
        rows = None
    else:
        heads = [(0, 0), (w.B - 1, w.H - 1)]
        rows = np.unique(np.concatenate([np.arange(0, 4), np.arange(w.L - 4, w.L),
                                         rng.choice(w.L, 24, replace=False)]))
    ref = oracle_heads(Q, K, V, w.causal, heads, rows=rows, two_pass=True, fp64=True)
    sel = (lambda a: a) if rows is None else (lambda a: a[rows])
    got = np.stack([sel(O[b, h]) for b, h in heads])
    online = np.stack([ref[k]["O"] for k in heads])
    two_pass = np.stack([ref[k]["O2"] for k in heads])
    fp64 = np.stack([ref[k]["Ox"] for k in heads])
    g_x, o_x, t_x = gap(got, fp64), gap(online, fp64), gap(two_pass, fp64)
    print(f"\n{w.name}: max-abs / aggregate relative error against fp64 attention -- "
          f"GPU {g_x[0]:.3e} / {g_x[1]:.3e}; oracle online {o_x[0]:.3e} / {o_x[1]:.3e}; "
          f"oracle two-pass {t_x[0]:.3e} / {t_x[1]:.3e}; GPU vs oracle online "
          f"{gap(got, online)[0]:.3e} / {gap(got, online)[1]:.3e}")
    assert g_x[1] <= 1.1 * o_x[1] + 1e-4
