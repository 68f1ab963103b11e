"""Write tests/golden/oracle_tiny.json: the CPU oracle's outputs on one tiny
seeded case (B=1, H=2, L=8, d=64, causal and non-causal).

Calls only the oracle (and the seeded input generator).  The stored values pin
the oracle against accidental change; the oracle itself is pinned by closed
forms in tests/test_oracle_*.py.  Rerun only when a change to the oracle's
arithmetic is justified by a passage of the pages:

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from int8_quantized_attention_token_b200.workloads import make_qkv  # noqa: E402


def main():
    Q, K, V = (t.float().numpy().reshape(2, 8, 64) for t in make_qkv(1, 2, 8, 64, seed=123))
    Qq, sQ = oracle.quantize_per_token(Q)
    Kq, sK = oracle.quantize_per_token(K)
    Vq, sV = oracle.quantize_per_tensor(V, 2)
    out = {
        "source": "IntAttention section 2.1 eqs. 3-5, section 2.2 eq. 6, section 3.2; "
                  "per-token Q/K after INT-FlashAttention's abstract",
        "case": {"B": 1, "H": 2, "L": 8, "d": 64, "seed": 123},
        "sQ": sQ.tolist(), "sK": sK.tolist(), "sV": sV.tolist(),
        "Qq_sum": int(Qq.astype(np.int64).sum()), "Kq_sum": int(Kq.astype(np.int64).sum()),
        "Vq_sum": int(Vq.astype(np.int64).sum()),
    }
    for causal in (False, True):
        O = oracle.attention_fwd(Qq, Kq, Vq, sQ, sK, sV, causal)
        out["O_causal" if causal else "O"] = [float(x) for x in O.ravel()]
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny.json"), "w") as f:
        json.dump(out, f)


if __name__ == "__main__":
    main()
