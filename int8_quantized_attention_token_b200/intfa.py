"""Thin ctypes binding of libintfa (include/intfa.h), same names as the C ABI.

Argument marshalling only: every step of the attention path runs in the CUDA
kernels of libintfa.so.  PyTorch supplies device memory and the current
stream.  There is no fallback: if the library is missing or a call fails, an
exception is raised.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libintfa.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "intfa.h")

STATUS = {0: "INTFA_OK", 1: "INTFA_ERR_INVALID_ARG", 2: "INTFA_ERR_UNSUPPORTED",
          3: "INTFA_ERR_MISALIGNED", 4: "INTFA_ERR_CUDA", 5: "INTFA_ERR_DEVICE_TIMEOUT",
          6: "INTFA_ERR_WORKSPACE"}


class IntfaError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {STATUS.get(code, code)} ({status_string(code)})")


_lib = None


def lib():
    """Load libintfa.so (built in-tree by ``build.build()``); raise if absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libintfa.so not built ({LIB_PATH}); run "
                           "python -m int8_quantized_attention_token_b200.build")
    L = ctypes.CDLL(LIB_PATH)
    P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    sig = {
        "intfa_status_string": ([I], ctypes.c_char_p),
        "intfa_quantize_per_token": ([P, I64, I, P, P, P], I),
        "intfa_quantize_per_token_bits": ([P, I64, I, I, P, P, P], I),
        "intfa_quantize_per_tensor_workspace_size": ([I64], SZ),
        "intfa_vt_ld": ([I64], I64),
        "intfa_quantize_per_tensor": ([P, I64, I64, I, I, P, P, P, SZ, P], I),
        "intfa_quantize_global": ([P, I64, I64, I, I, P, P, P, SZ, P], I),
        "intfa_quantize_per_tensor_noalloc": ([P, I64, I64, I, I, P, P, P], I),
        "intfa_attention_fwd": ([P, P, P, P, P, P, I, I, I, I, I, P, P], I),
        "intfa_attention_fwd_q16": ([P, P, P, P, P, I, I, I, I, I, P, P, P], I),
        "intfa_debug_qk": ([P, P, I, I, I, I, P, P], I),
        "intfa_attention_fwd_codesum": ([P, P, P, P, P, P, I, I, I, I, I, P, P], I),
        "intfa_attention_fwd_pcodes": ([P, P, P, P, P, P, I, I, I, I, I, I, I, P, P], I),
        "intfa_attention_fwd_blockscale": ([P, P, P, P, P, P, I, I, I, I, I, I, P, P], I),
        "intfa_decode_workspace_size": ([I, I, I, I], SZ),
        "intfa_decode_fwd": ([P, P, P, P, P, I, I, I, I, I, P, P, SZ, P], I),
        "intfa_index_attention_fwd": ([P, P, P, P, P, P, I, I, I, I, I, ctypes.c_double, I, P, P, P, P], I),
        "intfa_forward_workspace_size": ([I, I, I, I], SZ),
        "intfa_forward_workspace_layout": ([I, I, I, I, ctypes.POINTER(SZ)], I),
        "intfa_forward": ([P, P, P, I, I, I, I, I, P, P, SZ, P], I),
        "intfa_forward_host_workspace_size": ([I, I, I, I], SZ),
        "intfa_forward_host": ([P, P, P, I, I, I, I, I, P, P, SZ, P], I),
        "intfa_device_status": ([I, ctypes.POINTER(ctypes.c_uint32)], I),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    _lib = L
    return L


def declared_symbols() -> list[str]:
    """Entry points declared in include/intfa.h."""
    with open(HEADER_PATH) as f:
        text = f.read()
    return sorted(set(re.findall(r"\b(intfa_[a-z0-9_]+)\s*\(", text)))


def status_string(code: int) -> str:
    return lib().intfa_status_string(int(code)).decode()


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise IntfaError(rc, what)


def _stream(stream=None) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t) -> int:
    return t.data_ptr()


def _need(t: torch.Tensor, dtype, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


# ------------------------------------------------------------- entry points ---

def intfa_vt_ld(rows: int) -> int:
    return int(lib().intfa_vt_ld(int(rows)))


def intfa_quantize_per_token(x: torch.Tensor, x_q=None, scale=None, stream=None):
    """fp16 [..., d] -> (int8 [..., d], fp32 [...]); one scale per row."""
    _need(x, torch.float16, "x")
    d = x.shape[-1]
    rows = x.numel() // d if d else 0
    x_q = torch.empty(x.shape, dtype=torch.int8, device=x.device) if x_q is None else x_q
    scale = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device) if scale is None else scale
    _check(lib().intfa_quantize_per_token(_ptr(x), rows, d, _ptr(x_q), _ptr(scale), _stream(stream)),
           "intfa_quantize_per_token")
    return x_q, scale


def intfa_quantize_per_token_bits(x: torch.Tensor, bits: int, x_q=None, scale=None, stream=None):
    """fp16 [..., d] -> b-bit codes (in int8, |code| <= 2^(bits-1) - 1) and fp32 [...] scales."""
    _need(x, torch.float16, "x")
    d = x.shape[-1]
    rows = x.numel() // d if d else 0
    x_q = torch.empty(x.shape, dtype=torch.int8, device=x.device) if x_q is None else x_q
    scale = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device) if scale is None else scale
    _check(lib().intfa_quantize_per_token_bits(_ptr(x), rows, d, int(bits), _ptr(x_q), _ptr(scale), _stream(stream)),
           "intfa_quantize_per_token_bits")
    return x_q, scale


def intfa_quantize_per_tensor(x: torch.Tensor, transpose: bool = False, x_q=None, scale=None,
                              workspace=None, stream=None):
    """fp16 [groups, rows, cols] -> codes and fp32 [groups] scales.

    transpose=False: int8 [groups, rows, cols]; transpose=True: int8
    [groups, cols, intfa_vt_ld(rows)] (the V_hat^T layout of the attention)."""
    _need(x, torch.float16, "x")
    if x.dim() != 3:
        raise ValueError("x must be [groups, rows, cols]")
    g, rows, cols = x.shape
    if x_q is None:
        shape = (g, cols, intfa_vt_ld(rows)) if transpose else (g, rows, cols)
        x_q = torch.empty(shape, dtype=torch.int8, device=x.device)
    scale = torch.empty((g,), dtype=torch.float32, device=x.device) if scale is None else scale
    wsb = int(lib().intfa_quantize_per_tensor_workspace_size(g))
    if workspace is None:
        workspace = torch.empty((max(wsb, 1),), dtype=torch.uint8, device=x.device)
    _check(lib().intfa_quantize_per_tensor(_ptr(x), g, rows, cols, int(bool(transpose)), _ptr(x_q),
                                           _ptr(scale), _ptr(workspace), workspace.numel(),
                                           _stream(stream)), "intfa_quantize_per_tensor")
    return x_q, scale


def intfa_quantize_global(x: torch.Tensor, transpose: bool = False, x_q=None, scale=None, workspace=None,
                          stream=None):
    """fp16 [groups, rows, cols] -> codes with one scale over all groups (in
    the per-group layout of intfa_quantize_per_tensor) and fp32 [groups]
    scales, all equal."""
    _need(x, torch.float16, "x")
    if x.dim() != 3:
        raise ValueError("x must be [groups, rows, cols]")
    g, rows, cols = x.shape
    if x_q is None:
        shape = (g, cols, intfa_vt_ld(rows)) if transpose else (g, rows, cols)
        x_q = torch.empty(shape, dtype=torch.int8, device=x.device)
    scale = torch.empty((g,), dtype=torch.float32, device=x.device) if scale is None else scale
    wsb = int(lib().intfa_quantize_per_tensor_workspace_size(g))
    if workspace is None:
        workspace = torch.empty((max(wsb, 1),), dtype=torch.uint8, device=x.device)
    _check(lib().intfa_quantize_global(_ptr(x), g, rows, cols, int(bool(transpose)), _ptr(x_q), _ptr(scale),
                                       _ptr(workspace), workspace.numel(), _stream(stream)), "intfa_quantize_global")
    return x_q, scale


def intfa_quantize_per_tensor_noalloc(x: torch.Tensor, transpose: bool = False, x_q=None, scale=None,
                                      stream=None):
    """intfa_quantize_per_tensor without a workspace, for callers that cannot
    allocate device memory: the scratch is a fixed array inside the library
    (at most INTFA_NOALLOC_MAX_GROUPS = 4096 groups).  Calls that overlap on
    the GPU race on that array; the first call on a device does a one-time
    set-up and should come before any stream capture.  (This wrapper itself
    allocates outputs with torch when x_q / scale are not given.)"""
    _need(x, torch.float16, "x")
    if x.dim() != 3:
        raise ValueError("x must be [groups, rows, cols]")
    g, rows, cols = x.shape
    if x_q is None:
        shape = (g, cols, intfa_vt_ld(rows)) if transpose else (g, rows, cols)
        x_q = torch.empty(shape, dtype=torch.int8, device=x.device)
    scale = torch.empty((g,), dtype=torch.float32, device=x.device) if scale is None else scale
    _check(lib().intfa_quantize_per_tensor_noalloc(_ptr(x), g, rows, cols, int(bool(transpose)), _ptr(x_q),
                                                   _ptr(scale), _stream(stream)),
           "intfa_quantize_per_tensor_noalloc")
    return x_q, scale


def intfa_attention_fwd(Q_q, K_q, Vt_q, s_Q, s_K, s_V, causal: bool, O=None, stream=None):
    """Q_q, K_q int8 [B, H, L, d]; Vt_q int8 [B, H, d, intfa_vt_ld(L)];
    s_Q, s_K fp32 [B, H, L]; s_V fp32 [B, H]  ->  O fp16 [B, H, L, d]."""
    for t, n in ((Q_q, "Q_q"), (K_q, "K_q"), (Vt_q, "Vt_q")):
        _need(t, torch.int8, n)
    for t, n in ((s_Q, "s_Q"), (s_K, "s_K"), (s_V, "s_V")):
        _need(t, torch.float32, n)
    B, H, L, d = Q_q.shape
    O = torch.empty((B, H, L, d), dtype=torch.float16, device=Q_q.device) if O is None else O
    _check(lib().intfa_attention_fwd(_ptr(Q_q), _ptr(K_q), _ptr(Vt_q), _ptr(s_Q), _ptr(s_K),
                                     _ptr(s_V), B, H, L, d, int(bool(causal)), _ptr(O),
                                     _stream(stream)), "intfa_attention_fwd")
    return O


def intfa_attention_fwd_codesum(Q_q, K_q, Vt_q, s_Q, s_K, s_V, causal: bool, O=None, stream=None):
    """intfa_attention_fwd with the row sum taken from the P codes (sum P_hat / 127)."""
    for t, n in ((Q_q, "Q_q"), (K_q, "K_q"), (Vt_q, "Vt_q")):
        _need(t, torch.int8, n)
    for t, n in ((s_Q, "s_Q"), (s_K, "s_K"), (s_V, "s_V")):
        _need(t, torch.float32, n)
    B, H, L, d = Q_q.shape
    O = torch.empty((B, H, L, d), dtype=torch.float16, device=Q_q.device) if O is None else O
    _check(lib().intfa_attention_fwd_codesum(_ptr(Q_q), _ptr(K_q), _ptr(Vt_q), _ptr(s_Q), _ptr(s_K), _ptr(s_V),
                                             B, H, L, d, int(bool(causal)), _ptr(O), _stream(stream)),
           "intfa_attention_fwd_codesum")
    return O


def intfa_attention_fwd_pcodes(Q_q, K_q, Vt_q, s_Q, s_K, s_V, causal: bool, p_levels: int = 255,
                               lsum_codes: bool = False, O=None, stream=None):
    """intfa_attention_fwd with P codes RNE(p_levels p): 127 (INT8 P) or 255
    (UINT8 P); lsum_codes takes the row sum from the codes (sum P_hat / p_levels)."""
    for t, n in ((Q_q, "Q_q"), (K_q, "K_q"), (Vt_q, "Vt_q")):
        _need(t, torch.int8, n)
    for t, n in ((s_Q, "s_Q"), (s_K, "s_K"), (s_V, "s_V")):
        _need(t, torch.float32, n)
    B, H, L, d = Q_q.shape
    O = torch.empty((B, H, L, d), dtype=torch.float16, device=Q_q.device) if O is None else O
    _check(lib().intfa_attention_fwd_pcodes(_ptr(Q_q), _ptr(K_q), _ptr(Vt_q), _ptr(s_Q), _ptr(s_K), _ptr(s_V),
                                            B, H, L, d, int(bool(causal)), int(p_levels), int(bool(lsum_codes)),
                                            _ptr(O), _stream(stream)),
           "intfa_attention_fwd_pcodes")
    return O


def intfa_attention_fwd_blockscale(Q_q, K_q, Vt_q, s_Q, s_K, s_V, causal: bool, scale_block: int, O=None,
                                   stream=None):
    """intfa_attention_fwd with one Q / K scale per block of `scale_block`
    tokens: s_Q, s_K fp32 [B, H, ceil(L / scale_block)]."""
    for t, n in ((Q_q, "Q_q"), (K_q, "K_q"), (Vt_q, "Vt_q")):
        _need(t, torch.int8, n)
    for t, n in ((s_Q, "s_Q"), (s_K, "s_K"), (s_V, "s_V")):
        _need(t, torch.float32, n)
    B, H, L, d = Q_q.shape
    O = torch.empty((B, H, L, d), dtype=torch.float16, device=Q_q.device) if O is None else O
    _check(lib().intfa_attention_fwd_blockscale(_ptr(Q_q), _ptr(K_q), _ptr(Vt_q), _ptr(s_Q), _ptr(s_K),
                                                _ptr(s_V), B, H, L, d, int(bool(causal)), int(scale_block),
                                                _ptr(O), _stream(stream)), "intfa_attention_fwd_blockscale")
    return O


def intfa_attention_fwd_q16(Q, K_q, Vt_q, s_K, s_V, causal: bool, O=None, s_Q=None, stream=None):
    """Q fp16 [B, H, L, d] (quantised per token inside the kernel); K_q, Vt_q,
    s_K, s_V as for intfa_attention_fwd  ->  O fp16 [B, H, L, d].  If s_Q (fp32
    [B, H, L]) is given, the kernel writes Q's per-token scales into it."""
    _need(Q, torch.float16, "Q")
    for t, n in ((K_q, "K_q"), (Vt_q, "Vt_q")):
        _need(t, torch.int8, n)
    for t, n in ((s_K, "s_K"), (s_V, "s_V")):
        _need(t, torch.float32, n)
    if s_Q is not None:
        _need(s_Q, torch.float32, "s_Q")
    B, H, L, d = Q.shape
    O = torch.empty((B, H, L, d), dtype=torch.float16, device=Q.device) if O is None else O
    _check(lib().intfa_attention_fwd_q16(_ptr(Q), _ptr(K_q), _ptr(Vt_q), _ptr(s_K), _ptr(s_V), B, H, L, d,
                                         int(bool(causal)), _ptr(O), _ptr(s_Q) if s_Q is not None else None,
                                         _stream(stream)), "intfa_attention_fwd_q16")
    return O


def intfa_index_attention_fwd(Q_q, K_q, Vt_q, s_Q, s_K, s_V, causal: bool, c: float = 6.6, b: int = 5,
                              O=None, m_out=None, l_out=None, stream=None):
    """IndexSoftmax attention.  Q_q, K_q int8 [B, H, L, d] with per-head
    scales s_Q, s_K fp32 [B, H]; Vt_q int8 [B, H, d, intfa_vt_ld(L)] with s_V
    fp32 [B, H]; clip threshold c and table bits b  ->  O fp16 [B, H, L, d].
    m_out / l_out (int32 [B, H, L], optional) receive the integer row max of
    Q_hat K_hat^T and the integer row sum of the table values."""
    for t, n in ((Q_q, "Q_q"), (K_q, "K_q"), (Vt_q, "Vt_q")):
        _need(t, torch.int8, n)
    for t, n in ((s_Q, "s_Q"), (s_K, "s_K"), (s_V, "s_V")):
        _need(t, torch.float32, n)
    for t, n in ((m_out, "m_out"), (l_out, "l_out")):
        if t is not None:
            _need(t, torch.int32, n)
    B, H, L, d = Q_q.shape
    O = torch.empty((B, H, L, d), dtype=torch.float16, device=Q_q.device) if O is None else O
    _check(lib().intfa_index_attention_fwd(_ptr(Q_q), _ptr(K_q), _ptr(Vt_q), _ptr(s_Q), _ptr(s_K), _ptr(s_V),
                                           B, H, L, d, int(bool(causal)), float(c), int(b), _ptr(O),
                                           _ptr(m_out) if m_out is not None else None,
                                           _ptr(l_out) if l_out is not None else None,
                                           _stream(stream)), "intfa_index_attention_fwd")
    return O


def intfa_decode_fwd(q, K_q, s_K, V_q, s_V, splits: int = 1, O=None, workspace=None, stream=None):
    """One query per head against an INT8 cache: q fp16 [B, H, d]; K_q, V_q
    int8 [B, H, L, d] (per-token K codes, per-head V codes); s_K fp32 [B, H, L];
    s_V fp32 [B, H]  ->  O fp16 [B, H, d]."""
    _need(q, torch.float16, "q")
    for t, n in ((K_q, "K_q"), (V_q, "V_q")):
        _need(t, torch.int8, n)
    for t, n in ((s_K, "s_K"), (s_V, "s_V")):
        _need(t, torch.float32, n)
    B, H, L, d = K_q.shape
    O = torch.empty((B, H, d), dtype=torch.float16, device=q.device) if O is None else O
    wsb = int(lib().intfa_decode_workspace_size(B, H, d, int(splits)))
    if workspace is None:
        workspace = torch.empty((max(wsb, 16),), dtype=torch.uint8, device=q.device)
    _check(lib().intfa_decode_fwd(_ptr(q), _ptr(K_q), _ptr(s_K), _ptr(V_q), _ptr(s_V), B, H, L, d, int(splits),
                                  _ptr(O), _ptr(workspace), workspace.numel(), _stream(stream)),
           "intfa_decode_fwd")
    return O


def intfa_debug_qk(Q_q, K_q, S=None, stream=None):
    """int32 [B, H, L, L] = Q_hat K_hat^T through the tensor-core path."""
    _need(Q_q, torch.int8, "Q_q")
    _need(K_q, torch.int8, "K_q")
    B, H, L, d = Q_q.shape
    S = torch.empty((B, H, L, L), dtype=torch.int32, device=Q_q.device) if S is None else S
    _check(lib().intfa_debug_qk(_ptr(Q_q), _ptr(K_q), B, H, L, d, _ptr(S), _stream(stream)),
           "intfa_debug_qk")
    return S


def intfa_forward_workspace_size(B, H, L, d) -> int:
    return int(lib().intfa_forward_workspace_size(B, H, L, d))


def intfa_forward_host_workspace_size(B, H, L, d) -> int:
    return int(lib().intfa_forward_host_workspace_size(B, H, L, d))


def intfa_forward_workspace_layout(B, H, L, d) -> list[int]:
    off = (ctypes.c_size_t * 6)()
    _check(lib().intfa_forward_workspace_layout(B, H, L, d, off), "intfa_forward_workspace_layout")
    return list(off)


def intfa_forward(Q, K, V, causal: bool, O=None, workspace=None, stream=None):
    """fp16 [B, H, L, d] device tensors -> O fp16; quantisation + attention."""
    for t, n in ((Q, "Q"), (K, "K"), (V, "V")):
        _need(t, torch.float16, n)
    B, H, L, d = Q.shape
    O = torch.empty_like(Q) if O is None else O
    wsb = intfa_forward_workspace_size(B, H, L, d)
    if workspace is None:
        workspace = torch.empty((max(wsb, 1),), dtype=torch.uint8, device=Q.device)
    _check(lib().intfa_forward(_ptr(Q), _ptr(K), _ptr(V), B, H, L, d, int(bool(causal)), _ptr(O),
                               _ptr(workspace), workspace.numel(), _stream(stream)), "intfa_forward")
    return O


def intfa_forward_host(Q_host, K_host, V_host, causal: bool, O_host, workspace, stream=None):
    """Host (pinned) fp16 tensors in and out; copies run inside the call."""
    for t, n in ((Q_host, "Q"), (K_host, "K"), (V_host, "V"), (O_host, "O")):
        if t.is_cuda or t.dtype != torch.float16 or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous fp16 host tensor")
    B, H, L, d = Q_host.shape
    _check(lib().intfa_forward_host(_ptr(Q_host), _ptr(K_host), _ptr(V_host), B, H, L, d,
                                    int(bool(causal)), _ptr(O_host), _ptr(workspace),
                                    workspace.numel(), _stream(stream)), "intfa_forward_host")
    return O_host


def intfa_device_status(clear: bool = True) -> int:
    """Synchronise and return the device status word (0 = no kernel timed out)."""
    w = ctypes.c_uint32(0)
    rc = lib().intfa_device_status(int(bool(clear)), ctypes.byref(w))
    if rc not in (0, 5):
        raise IntfaError(rc, "intfa_device_status")
    return int(w.value)
