"""CPU oracle for the INT8-quantised attention forward pass.

TEST INFRASTRUCTURE: only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg import this package.  The product
path (the CUDA library and its Python binding) never imports or calls it.

The arithmetic lives in ``oracle.c`` (plain C, fp64 for the softmax and the
value path, IEEE fp32 for the quantiser); this module only builds it with gcc
and marshals numpy arrays.  Each function cites the passage it follows:

* ``quantize_per_token`` / ``quantize_per_tensor`` -- IntAttention (A Fully
  Integer Attention Pipeline for Efficient Edge Inference), section 2.1,
  eq. 3; per-token granularity from INT-FlashAttention (Enabling Flash
  Attention for INT8 Quantization), abstract.
* ``qk_int32`` -- IntAttention section 2.1, eq. 4 (INT8 x INT8 -> INT32).
* ``attention_rows`` -- IntAttention eqs. 4-6 and section 3.2 (P x 127 as
  INT8), eq. 5 for the value path; two passes, P codes against the final
  row max.
* ``attention_online_rows`` -- the same steps in FlashAttention's block-wise
  online order (INT-FlashAttention abstract; FlashAttention-3 abstract): P
  codes against the running max of the key blocks seen so far.  This is the
  form the fused kernel computes.  ``p_levels=255`` stores P as UINT8
  (RNE(255 p)), the unsigned scheme of IntAttention's Table 5 ablation.
* ``attention_fp64_rows`` -- IntAttention section 2.1, eq. 1.
* ``decode`` -- one query against a key / value cache: the online form of
  ``attention_online_rows`` run separately on consecutive key ranges
  (split-KV) and merged (FlashAttention's block-wise softmax at range level).
* ``index_lut``, ``index_cint``, ``index_attention_rows`` -- IntAttention
  sections 3.1-3.2 (IndexSoftmax: eqs. 7-10, the UINT8 exponential table,
  UINT8 P times 255, integer row sums) with per-tensor Q / K scales
  (section 3.3's default configuration).

All functions are pinned by ``tests/test_oracle_*.py`` (closed forms,
invariants, brute force on tiny inputs).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into oracle/liboracle.so with plain gcc (no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", _LIB_PATH, "-lm"]
        subprocess.check_call(cmd)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB_PATH)
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    lib.oracle_set_threads.argtypes = [ctypes.c_int]
    lib.oracle_get_threads.restype = ctypes.c_int
    lib.oracle_quantize_per_token.argtypes = [P, I64, I64, P, P]
    lib.oracle_quantize_per_tensor.argtypes = [P, I64, I64, P, P]
    lib.oracle_quantize_per_token_bits.argtypes = [P, I64, I64, ctypes.c_int, P, P]
    lib.oracle_qk_int32.argtypes = [P, P, I64, I64, I64, P]
    lib.oracle_attention_rows.argtypes = [P, P, P, P, P, ctypes.c_float, I64, I64,
                                          ctypes.c_int, I64, I64, P, P, P, P]
    lib.oracle_attention_online_rows.argtypes = [P, P, P, P, P, ctypes.c_float, I64, I64,
                                                 ctypes.c_int, I64, I64, I64, P, P, ctypes.c_int, ctypes.c_int]
    lib.oracle_attention_fp64_rows.argtypes = [P, P, P, I64, I64, ctypes.c_int, I64, I64, P]
    lib.oracle_decode.argtypes = [P, ctypes.c_float, P, P, P, ctypes.c_float, I64, I64, I64, I64, P]
    lib.oracle_index_lut.argtypes = [ctypes.c_double, ctypes.c_int, P]
    lib.oracle_index_cint.argtypes = [ctypes.c_double, I64, ctypes.c_float, ctypes.c_float]
    lib.oracle_index_cint.restype = I64
    lib.oracle_index_attention_rows.argtypes = [P, P, P, ctypes.c_float, ctypes.c_float,
                                                ctypes.c_float, I64, I64, ctypes.c_int,
                                                ctypes.c_double, ctypes.c_int, I64, I64,
                                                P, P, P, P]
    _lib = lib
    return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(_load().oracle_get_threads())


def quantize_per_token(x):
    """x: float32 [..., d] (exact widening of fp16).  Returns (int8 [..., d], fp32 [...])."""
    x = _c(x, np.float32)
    d = x.shape[-1]
    rows = x.size // d if d else 0
    q = np.empty(x.shape, np.int8)
    s = np.empty(x.shape[:-1], np.float32)
    _load().oracle_quantize_per_token(_ptr(x), rows, d, _ptr(q), _ptr(s))
    return q, s


def quantize_per_token_bits(x, bits: int):
    """x: float32 [..., d]; b-bit symmetric codes (qmax = 2^(b-1) - 1) in int8
    and fp32 scales max|x| / qmax per row."""
    if not 2 <= bits <= 8:
        raise ValueError("bits in 2..8")
    x = _c(x, np.float32)
    d = x.shape[-1]
    rows = x.size // d if d else 0
    q = np.empty(x.shape, np.int8)
    s = np.empty(x.shape[:-1], np.float32)
    _load().oracle_quantize_per_token_bits(_ptr(x), rows, d, int(bits), _ptr(q), _ptr(s))
    return q, s


def quantize_per_tensor(x, groups: int):
    """x: float32 with x.size divisible by groups; one scale per contiguous group."""
    x = _c(x, np.float32)
    n = x.size // groups
    q = np.empty(x.shape, np.int8)
    s = np.empty((groups,), np.float32)
    _load().oracle_quantize_per_tensor(_ptr(x), groups, n, _ptr(q), _ptr(s))
    return q, s


def qk_int32(Qq, Kq):
    """Qq, Kq: int8 [heads, L, d].  Returns int32 [heads, L, L]."""
    Qq = _c(Qq, np.int8)
    Kq = _c(Kq, np.int8)
    heads, L, d = Qq.shape
    S = np.empty((heads, L, L), np.int32)
    _load().oracle_qk_int32(_ptr(Qq), _ptr(Kq), heads, L, d, _ptr(S))
    return S


def attention_rows(Qq, Kq, Vq, sQ, sK, sV: float, causal: bool, r0: int = 0, r1=None,
                   want_stats: bool = False, want_P: bool = False):
    """One head: Qq/Kq/Vq int8 [L, d], sQ/sK fp32 [L], sV the head's scale.

    Returns O fp64 [r1 - r0, d]; with want_stats also (m, l); with want_P also
    the int32 P codes [r1 - r0, L]."""
    Qq = _c(Qq, np.int8)
    Kq = _c(Kq, np.int8)
    Vq = _c(Vq, np.int8)
    sQ = _c(sQ, np.float32)
    sK = _c(sK, np.float32)
    L, d = Qq.shape
    r1 = L if r1 is None else r1
    n = r1 - r0
    O = np.empty((n, d), np.float64)
    m = np.empty((n,), np.float64) if want_stats else None
    l = np.empty((n,), np.float64) if want_stats else None
    P = np.empty((n, L), np.int32) if want_P else None
    _load().oracle_attention_rows(_ptr(Qq), _ptr(Kq), _ptr(Vq), _ptr(sQ), _ptr(sK),
                                  float(sV), L, d, int(bool(causal)), r0, r1,
                                  _ptr(O), _ptr(m), _ptr(l), _ptr(P))
    out = [O]
    if want_stats:
        out += [m, l]
    if want_P:
        out.append(P)
    return out[0] if len(out) == 1 else tuple(out)


def attention_online_rows(Qq, Kq, Vq, sQ, sK, sV: float, causal: bool, block: int = 128,
                          r0: int = 0, r1=None, want_l: bool = False, lsum_codes: bool = False,
                          p_levels: int = 127):
    """One head, block-wise online form (FlashAttention's forward workflow):
    P codes against the running max over key blocks of ``block``.  Returns O
    fp64 [r1 - r0, d] (and the row sums l with want_l).  lsum_codes: the row
    sum from the P codes (sum P_hat / p_levels) instead of the unquantised p.
    p_levels: 127 (P codes RNE(127 p), INT8) or 255 (RNE(255 p), UINT8 --
    IntAttention Table 5's unsigned scheme)."""
    if p_levels not in (127, 255):
        raise ValueError("p_levels must be 127 or 255")
    Qq = _c(Qq, np.int8)
    Kq = _c(Kq, np.int8)
    Vq = _c(Vq, np.int8)
    sQ = _c(sQ, np.float32)
    sK = _c(sK, np.float32)
    L, d = Qq.shape
    r1 = L if r1 is None else r1
    O = np.empty((r1 - r0, d), np.float64)
    l = np.empty((r1 - r0,), np.float64) if want_l else None
    _load().oracle_attention_online_rows(_ptr(Qq), _ptr(Kq), _ptr(Vq), _ptr(sQ), _ptr(sK),
                                         float(sV), L, d, int(bool(causal)), int(block),
                                         r0, r1, _ptr(O), _ptr(l), int(bool(lsum_codes)), int(p_levels))
    return (O, l) if want_l else O


def attention_fp64_rows(Q, K, V, causal: bool, r0: int = 0, r1=None):
    """One head, unquantised: Q/K/V float32 [L, d].  Returns fp64 [r1 - r0, d]."""
    Q = _c(Q, np.float32)
    K = _c(K, np.float32)
    V = _c(V, np.float32)
    L, d = Q.shape
    r1 = L if r1 is None else r1
    O = np.empty((r1 - r0, d), np.float64)
    _load().oracle_attention_fp64_rows(_ptr(Q), _ptr(K), _ptr(V), L, d, int(bool(causal)),
                                       r0, r1, _ptr(O))
    return O


def attention_fwd(Qq, Kq, Vq, sQ, sK, sV, causal: bool):
    """All heads: Qq/Kq/Vq int8 [BH, L, d] (V_hat row-major, not transposed),
    sQ/sK fp32 [BH, L], sV fp32 [BH].  Returns O fp64 [BH, L, d]."""
    BH, L, d = Qq.shape
    O = np.empty((BH, L, d), np.float64)
    for h in range(BH):
        O[h] = attention_rows(Qq[h], Kq[h], Vq[h], sQ[h], sK[h], float(sV[h]), causal)
    return O


def attention_online_fwd(Qq, Kq, Vq, sQ, sK, sV, causal: bool, block: int = 128):
    """All heads, block-wise online form: int8 [BH, L, d] -> fp64 [BH, L, d]."""
    BH, L, d = Qq.shape
    O = np.empty((BH, L, d), np.float64)
    for h in range(BH):
        O[h] = attention_online_rows(Qq[h], Kq[h], Vq[h], sQ[h], sK[h], float(sV[h]), causal, block)
    return O


def attention_fp64(Q, K, V, causal: bool):
    """All heads, unquantised: float32 [BH, L, d] -> fp64 [BH, L, d]."""
    BH, L, d = Q.shape
    O = np.empty((BH, L, d), np.float64)
    for h in range(BH):
        O[h] = attention_fp64_rows(Q[h], K[h], V[h], causal)
    return O


# ---------------------------------------------------------------- IndexSoftmax

INDEX_C = 6.6   # IntAttention ablation (Fig. 9): the recommended (b, c) = (5, 6.6)
INDEX_B = 5


def index_lut(c: float = INDEX_C, b: int = INDEX_B):
    """The 2^b-entry UINT8 exponential table: RNE(255 exp(-c k / (2^b - 1)))."""
    if not 1 <= b <= 8:
        raise ValueError("b in 1..8")
    lut = np.empty((1 << b,), np.uint8)
    _load().oracle_index_lut(float(c), int(b), _ptr(lut))
    return lut


def index_cint(c: float, d: int, sQ: float, sK: float) -> int:
    """c_int = rint(c sqrt(d) / (s_Q s_K)) in fp64, at least 1 (eq. 8)."""
    return int(_load().oracle_index_cint(float(c), int(d), float(sQ), float(sK)))


def index_attention_rows(Qq, Kq, Vq, sQ: float, sK: float, sV: float, causal: bool,
                         c: float = INDEX_C, b: int = INDEX_B, r0: int = 0, r1=None,
                         want_stats: bool = False, want_E: bool = False):
    """One head of IndexSoftmax attention: Qq/Kq/Vq int8 [L, d] with per-tensor
    scales.  Returns O fp64 [r1 - r0, d]; with want_stats also the integer row
    max of Q_hat K_hat^T and the integer row sum of E (int64); with want_E the
    UINT8 table values E [r1 - r0, L] (0 for masked keys)."""
    if not 1 <= b <= 8:
        raise ValueError("b in 1..8")
    Qq = _c(Qq, np.int8)
    Kq = _c(Kq, np.int8)
    Vq = _c(Vq, np.int8)
    L, d = Qq.shape
    r1 = L if r1 is None else r1
    n = r1 - r0
    O = np.empty((n, d), np.float64)
    m = np.empty((n,), np.int64) if want_stats else None
    l = np.empty((n,), np.int64) if want_stats else None
    E = np.empty((n, L), np.int32) if want_E else None
    _load().oracle_index_attention_rows(_ptr(Qq), _ptr(Kq), _ptr(Vq), float(sQ), float(sK),
                                        float(sV), L, d, int(bool(causal)), float(c), int(b),
                                        r0, r1, _ptr(O), _ptr(m), _ptr(l), _ptr(E))
    out = [O]
    if want_stats:
        out += [m, l]
    if want_E:
        out.append(E)
    return out[0] if len(out) == 1 else tuple(out)


def index_attention_fwd(Qq, Kq, Vq, sQ, sK, sV, causal: bool, c: float = INDEX_C,
                        b: int = INDEX_B, want_stats: bool = False):
    """All heads: int8 [BH, L, d] (V_hat row-major), per-head scales fp32
    [BH] for Q, K and V.  Returns O fp64 [BH, L, d] (and int64 m, l [BH, L]
    with want_stats)."""
    BH, L, d = Qq.shape
    O = np.empty((BH, L, d), np.float64)
    M = np.empty((BH, L), np.int64)
    Ls = np.empty((BH, L), np.int64)
    for h in range(BH):
        O[h], M[h], Ls[h] = index_attention_rows(Qq[h], Kq[h], Vq[h], float(sQ[h]), float(sK[h]),
                                                 float(sV[h]), causal, c, b, want_stats=True)
    return (O, M, Ls) if want_stats else O


# ---------------------------------------------------------------- decode

def decode(q, sq: float, Kq, sK, Vq, sV: float, block: int = 128, split_len=None):
    """One query: q int8 [d] (scale sq), Kq / Vq int8 [L, d], sK fp32 [L], sV
    the cache's value scale.  Keys in ranges of split_len (a multiple of
    block; default: one range).  Returns O fp64 [d]."""
    q = _c(q, np.int8)
    Kq = _c(Kq, np.int8)
    Vq = _c(Vq, np.int8)
    sK = _c(sK, np.float32)
    L, d = Kq.shape
    split_len = -(-L // block) * block if split_len is None else int(split_len)
    if split_len % block:
        raise ValueError("split_len must be a multiple of block")
    O = np.empty((d,), np.float64)
    _load().oracle_decode(_ptr(q), float(sq), _ptr(Kq), _ptr(sK), _ptr(Vq), float(sV), L, d, int(block),
                          max(split_len, block), _ptr(O))
    return O
