"""Helpers shared by the GPU parity tests: run the CPU oracle on the same
seeded fp16 inputs (it quantises them itself) and measure the gap."""
import numpy as np
import torch

import oracle


def oracle_heads(Q, K, V, causal, heads, rows=None, two_pass=False, fp64=False, block=128,
                 p_levels=127, lsum_codes=False):
    """Q, K, V: fp16 CPU [B, H, L, d].  For each (b, h) in heads, quantise that
    head with the oracle and run the online form (P codes RNE(p_levels p),
    row sum from the codes with lsum_codes; optionally also the two-pass form
    and unquantised fp64 attention) on `rows` (all rows if None).
    Returns {(b, h): dict(rows=..., O=..., O2=..., Ox=...)}."""
    out = {}
    L = Q.shape[2]
    for (b, h) in heads:
        q = Q[b, h].float().numpy()
        k = K[b, h].float().numpy()
        v = V[b, h].float().numpy()
        Qq, sQ = oracle.quantize_per_token(q)
        Kq, sK = oracle.quantize_per_token(k)
        Vq, sV = oracle.quantize_per_tensor(v, 1)
        rr = np.arange(L) if rows is None else np.asarray(rows)
        res = {"rows": rr, "O": np.empty((len(rr), q.shape[1]))}
        if two_pass:
            res["O2"] = np.empty_like(res["O"])
        if fp64:
            res["Ox"] = np.empty_like(res["O"])
        # contiguous runs of rows in one call each
        start = 0
        while start < len(rr):
            stop = start + 1
            while stop < len(rr) and rr[stop] == rr[stop - 1] + 1:
                stop += 1
            r0, r1 = int(rr[start]), int(rr[stop - 1]) + 1
            res["O"][start:stop] = oracle.attention_online_rows(Qq, Kq, Vq, sQ, sK, float(sV[0]),
                                                                causal, block, r0, r1,
                                                                lsum_codes=lsum_codes, p_levels=p_levels)
            if two_pass:
                res["O2"][start:stop] = oracle.attention_rows(Qq, Kq, Vq, sQ, sK, float(sV[0]),
                                                              causal, r0, r1)
            if fp64:
                res["Ox"][start:stop] = oracle.attention_fp64_rows(q, k, v, causal, r0, r1)
            start = stop
        out[(b, h)] = res
    return out


def gap(O, ref):
    """(max|O - ref| / max|ref|, sum|O - ref| / sum|ref|)."""
    O = np.asarray(O, np.float64)
    ref = np.asarray(ref, np.float64)
    d = np.abs(O - ref)
    return float(d.max() / np.abs(ref).max()), float(d.sum() / np.abs(ref).sum())


# Tolerances for the fp16 output against the oracle's block-wise online form
# (the same algorithm in fp64): max-abs <= 1e-2 max|O| and aggregate relative
# error <= 2e-3.
TOL_MAXABS = 1e-2
TOL_MRE = 2e-3
