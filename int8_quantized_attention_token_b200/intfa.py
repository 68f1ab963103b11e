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
        "intfa_attention_fwd_vrows": ([P, P, P, P, P, P, I, I, I, I, I, P, P], I),
        "intfa_attention_fwd_q16": ([P, P, P, P, P, I, I, I, I, I, P, P, P], I),
        "intfa_debug_qk": ([P, P, I, I, I, I, P, P], I),
        "intfa_debug_attention_scores": ([P, P, P, P, P, P, I, I, I, I, I, P, P, P], I),
        "intfa_debug_wait_timeout": ([P, P, P, P, P, P, I, I, I, I, I, P, I64, P], I),
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


def _need(t: torch.Tensor, dtype, name: str, shape=None, device=None):
    """t must be a contiguous CUDA tensor of `dtype` (and of `shape` / on
    `device` when given): the library writes through raw pointers, so a wrong
    size or a tensor on another GPU must be caught before any launch."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def _out(t, shape, dtype, device, name: str):
    """A caller-provided output (checked like an input), or a new tensor."""
    if t is None:
        return torch.empty(tuple(shape), dtype=dtype, device=device)
    _need(t, dtype, name, shape=shape, device=device)
    return t


def _on(device):
    """The library launches on the current CUDA device: make it x's."""
    return torch.cuda.device(device)


# ------------------------------------------------------------- entry points ---

def intfa_vt_ld(rows: int) -> int:
    return int(lib().intfa_vt_ld(int(rows)))


def intfa_quantize_per_token(x: torch.Tensor, x_q=None, scale=None, stream=None):
    """fp16 [..., d] -> (int8 [..., d], fp32 [...]); one scale per row."""
    _need(x, torch.float16, "x")
    d = x.shape[-1]
    rows = x.numel() // d if d else 0
    x_q = _out(x_q, x.shape, torch.int8, x.device, "x_q")
    scale = _out(scale, x.shape[:-1], torch.float32, x.device, "scale")
    with _on(x.device):
        _check(lib().intfa_quantize_per_token(_ptr(x), rows, d, _ptr(x_q), _ptr(scale), _stream(stream)),
               "intfa_quantize_per_token")
    return x_q, scale


def intfa_quantize_per_token_bits(x: torch.Tensor, bits: int, x_q=None, scale=None, stream=None):
    """fp16 [..., d] -> b-bit codes (in int8, |code| <= 2^(bits-1) - 1) and fp32 [...] scales."""
    _need(x, torch.float16, "x")
    d = x.shape[-1]
    rows = x.numel() // d if d else 0
    x_q = _out(x_q, x.shape, torch.int8, x.device, "x_q")
    scale = _out(scale, x.shape[:-1], torch.float32, x.device, "scale")
    with _on(x.device):
        _check(lib().intfa_quantize_per_token_bits(_ptr(x), rows, d, int(bits), _ptr(x_q), _ptr(scale),
                                                   _stream(stream)), "intfa_quantize_per_token_bits")
    return x_q, scale


def _tensor_outputs(x, transpose, x_q, scale):
    """Codes ([g, rows, cols], or [g, cols, intfa_vt_ld(rows)] transposed)
    and the g scales of a per-tensor quantisation of x [g, rows, cols]."""
    g, rows, cols = x.shape
    shape = (g, cols, intfa_vt_ld(rows)) if transpose else (g, rows, cols)
    return (_out(x_q, shape, torch.int8, x.device, "x_q"),
            _out(scale, (g,), torch.float32, x.device, "scale"))


def _workspace(ws, nbytes, device):
    if ws is None:
        return torch.empty((max(nbytes, 1),), dtype=torch.uint8, device=device)
    _need(ws, torch.uint8, "workspace", device=device)
    if ws.numel() < nbytes:
        raise ValueError(f"workspace must hold {nbytes} bytes, got {ws.numel()}")
    return ws


def intfa_quantize_per_tensor(x: torch.Tensor, transpose: bool = False, x_q=None, scale=None,
                              workspace=None, stream=None):
    """fp16 [groups, rows, cols] -> codes and fp32 [groups] scales.

    transpose=False: int8 [groups, rows, cols]; transpose=True: int8
    [groups, cols, intfa_vt_ld(rows)] (the V_hat^T layout of the attention)."""
    _need(x, torch.float16, "x")
    if x.dim() != 3:
        raise ValueError("x must be [groups, rows, cols]")
    g, rows, cols = x.shape
    x_q, scale = _tensor_outputs(x, transpose, x_q, scale)
    workspace = _workspace(workspace, int(lib().intfa_quantize_per_tensor_workspace_size(g)), x.device)
    with _on(x.device):
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
    x_q, scale = _tensor_outputs(x, transpose, x_q, scale)
    workspace = _workspace(workspace, int(lib().intfa_quantize_per_tensor_workspace_size(g)), x.device)
    with _on(x.device):
        _check(lib().intfa_quantize_global(_ptr(x), g, rows, cols, int(bool(transpose)), _ptr(x_q), _ptr(scale),
                                           _ptr(workspace), workspace.numel(), _stream(stream)),
               "intfa_quantize_global")
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
    x_q, scale = _tensor_outputs(x, transpose, x_q, scale)
    with _on(x.device):
        _check(lib().intfa_quantize_per_tensor_noalloc(_ptr(x), g, rows, cols, int(bool(transpose)), _ptr(x_q),
                                                       _ptr(scale), _stream(stream)),
               "intfa_quantize_per_tensor_noalloc")
    return x_q, scale


def _attn_inputs(Q_q, K_q, Vt_q, s_Q, s_K, s_V, nsc=None, vrows=False):
    """Check the fused attention's inputs against Q_q's shape [B, H, L, d] and
    device; nsc = scales per head of s_Q / s_K (L unless per-block); vrows:
    V_hat as [B, H, L, d] rather than transposed."""
    if not isinstance(Q_q, torch.Tensor) or Q_q.dim() != 4:
        raise ValueError("Q_q must be [B, H, L, d]")
    B, H, L, d = Q_q.shape
    dev = Q_q.device
    nsc = L if nsc is None else nsc
    _need(Q_q, torch.int8, "Q_q", device=dev)
    _need(K_q, torch.int8, "K_q", shape=(B, H, L, d), device=dev)
    if vrows:
        _need(Vt_q, torch.int8, "V_q", shape=(B, H, L, d), device=dev)
    else:
        _need(Vt_q, torch.int8, "Vt_q", shape=(B, H, d, intfa_vt_ld(L)), device=dev)
    _need(s_Q, torch.float32, "s_Q", shape=(B, H, nsc), device=dev)
    _need(s_K, torch.float32, "s_K", shape=(B, H, nsc), device=dev)
    _need(s_V, torch.float32, "s_V", shape=(B, H), device=dev)
    return B, H, L, d


def intfa_attention_fwd(Q_q, K_q, Vt_q, s_Q, s_K, s_V, causal: bool, O=None, stream=None):
    """Q_q, K_q int8 [B, H, L, d]; Vt_q int8 [B, H, d, intfa_vt_ld(L)];
    s_Q, s_K fp32 [B, H, L]; s_V fp32 [B, H]  ->  O fp16 [B, H, L, d]."""
    B, H, L, d = _attn_inputs(Q_q, K_q, Vt_q, s_Q, s_K, s_V)
    O = _out(O, (B, H, L, d), torch.float16, Q_q.device, "O")
    with _on(Q_q.device):
        _check(lib().intfa_attention_fwd(_ptr(Q_q), _ptr(K_q), _ptr(Vt_q), _ptr(s_Q), _ptr(s_K),
                                         _ptr(s_V), B, H, L, d, int(bool(causal)), _ptr(O),
                                         _stream(stream)), "intfa_attention_fwd")
    return O


def intfa_attention_fwd_vrows(Q_q, K_q, V_q, s_Q, s_K, s_V, causal: bool, O=None, stream=None):
    """intfa_attention_fwd with V_q int8 [B, H, L, d] (V_hat untransposed)."""
    B, H, L, d = _attn_inputs(Q_q, K_q, V_q, s_Q, s_K, s_V, vrows=True)
    O = _out(O, (B, H, L, d), torch.float16, Q_q.device, "O")
    with _on(Q_q.device):
        _check(lib().intfa_attention_fwd_vrows(_ptr(Q_q), _ptr(K_q), _ptr(V_q), _ptr(s_Q), _ptr(s_K),
                                               _ptr(s_V), B, H, L, d, int(bool(causal)), _ptr(O),
                                               _stream(stream)), "intfa_attention_fwd_vrows")
    return O


def intfa_attention_fwd_codesum(Q_q, K_q, Vt_q, s_Q, s_K, s_V, causal: bool, O=None, stream=None):
    """intfa_attention_fwd with the row sum taken from the P codes (sum P_hat / 127)."""
    B, H, L, d = _attn_inputs(Q_q, K_q, Vt_q, s_Q, s_K, s_V)
    O = _out(O, (B, H, L, d), torch.float16, Q_q.device, "O")
    with _on(Q_q.device):
        _check(lib().intfa_attention_fwd_codesum(_ptr(Q_q), _ptr(K_q), _ptr(Vt_q), _ptr(s_Q), _ptr(s_K), _ptr(s_V),
                                                 B, H, L, d, int(bool(causal)), _ptr(O), _stream(stream)),
               "intfa_attention_fwd_codesum")
    return O


def intfa_attention_fwd_pcodes(Q_q, K_q, Vt_q, s_Q, s_K, s_V, causal: bool, p_levels: int = 255,
                               lsum_codes: bool = False, O=None, stream=None):
    """intfa_attention_fwd with P codes RNE(p_levels p): 127 (INT8 P) or 255
    (UINT8 P); lsum_codes takes the row sum from the codes (sum P_hat / p_levels)."""
    B, H, L, d = _attn_inputs(Q_q, K_q, Vt_q, s_Q, s_K, s_V)
    O = _out(O, (B, H, L, d), torch.float16, Q_q.device, "O")
    with _on(Q_q.device):
        _check(lib().intfa_attention_fwd_pcodes(_ptr(Q_q), _ptr(K_q), _ptr(Vt_q), _ptr(s_Q), _ptr(s_K), _ptr(s_V),
                                                B, H, L, d, int(bool(causal)), int(p_levels), int(bool(lsum_codes)),
                                                _ptr(O), _stream(stream)),
               "intfa_attention_fwd_pcodes")
    return O


def intfa_attention_fwd_blockscale(Q_q, K_q, Vt_q, s_Q, s_K, s_V, causal: bool, scale_block: int, O=None,
                                   stream=None):
    """intfa_attention_fwd with one Q / K scale per block of `scale_block`
    tokens: s_Q, s_K fp32 [B, H, ceil(L / scale_block)]."""
    L0 = Q_q.shape[2] if isinstance(Q_q, torch.Tensor) and Q_q.dim() == 4 else 0
    sb = max(int(scale_block), 1)
    B, H, L, d = _attn_inputs(Q_q, K_q, Vt_q, s_Q, s_K, s_V, nsc=(L0 + sb - 1) // sb)
    O = _out(O, (B, H, L, d), torch.float16, Q_q.device, "O")
    with _on(Q_q.device):
        _check(lib().intfa_attention_fwd_blockscale(_ptr(Q_q), _ptr(K_q), _ptr(Vt_q), _ptr(s_Q), _ptr(s_K),
                                                    _ptr(s_V), B, H, L, d, int(bool(causal)), int(scale_block),
                                                    _ptr(O), _stream(stream)), "intfa_attention_fwd_blockscale")
    return O


def intfa_attention_fwd_q16(Q, K_q, Vt_q, s_K, s_V, causal: bool, O=None, s_Q=None, stream=None):
    """Q fp16 [B, H, L, d] (quantised per token inside the kernel); K_q, Vt_q,
    s_K, s_V as for intfa_attention_fwd  ->  O fp16 [B, H, L, d].  If s_Q (fp32
    [B, H, L]) is given, the kernel writes Q's per-token scales into it."""
    if not isinstance(Q, torch.Tensor) or Q.dim() != 4:
        raise ValueError("Q must be [B, H, L, d]")
    B, H, L, d = Q.shape
    dev = Q.device
    _need(Q, torch.float16, "Q", device=dev)
    _need(K_q, torch.int8, "K_q", shape=(B, H, L, d), device=dev)
    _need(Vt_q, torch.int8, "Vt_q", shape=(B, H, d, intfa_vt_ld(L)), device=dev)
    _need(s_K, torch.float32, "s_K", shape=(B, H, L), device=dev)
    _need(s_V, torch.float32, "s_V", shape=(B, H), device=dev)
    if s_Q is not None:
        _need(s_Q, torch.float32, "s_Q", shape=(B, H, L), device=dev)
    O = _out(O, (B, H, L, d), torch.float16, dev, "O")
    with _on(dev):
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
    if not isinstance(Q_q, torch.Tensor) or Q_q.dim() != 4:
        raise ValueError("Q_q must be [B, H, L, d]")
    B, H, L, d = Q_q.shape
    dev = Q_q.device
    _need(Q_q, torch.int8, "Q_q", device=dev)
    _need(K_q, torch.int8, "K_q", shape=(B, H, L, d), device=dev)
    _need(Vt_q, torch.int8, "Vt_q", shape=(B, H, d, intfa_vt_ld(L)), device=dev)
    for t, n in ((s_Q, "s_Q"), (s_K, "s_K"), (s_V, "s_V")):
        _need(t, torch.float32, n, shape=(B, H), device=dev)
    for t, n in ((m_out, "m_out"), (l_out, "l_out")):
        if t is not None:
            _need(t, torch.int32, n, shape=(B, H, L), device=dev)
    O = _out(O, (B, H, L, d), torch.float16, dev, "O")
    with _on(dev):
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
    if not isinstance(K_q, torch.Tensor) or K_q.dim() != 4:
        raise ValueError("K_q must be [B, H, L, d]")
    B, H, L, d = K_q.shape
    dev = K_q.device
    _need(q, torch.float16, "q", shape=(B, H, d), device=dev)
    _need(K_q, torch.int8, "K_q", device=dev)
    _need(V_q, torch.int8, "V_q", shape=(B, H, L, d), device=dev)
    _need(s_K, torch.float32, "s_K", shape=(B, H, L), device=dev)
    _need(s_V, torch.float32, "s_V", shape=(B, H), device=dev)
    O = _out(O, (B, H, d), torch.float16, dev, "O")
    workspace = _workspace(workspace, int(lib().intfa_decode_workspace_size(B, H, d, int(splits))), dev)
    with _on(dev):
        _check(lib().intfa_decode_fwd(_ptr(q), _ptr(K_q), _ptr(s_K), _ptr(V_q), _ptr(s_V), B, H, L, d,
                                      int(splits), _ptr(O), _ptr(workspace), workspace.numel(), _stream(stream)),
               "intfa_decode_fwd")
    return O


def intfa_debug_qk(Q_q, K_q, S=None, stream=None):
    """int32 [B, H, L, L] = Q_hat K_hat^T through the tensor-core path."""
    if not isinstance(Q_q, torch.Tensor) or Q_q.dim() != 4:
        raise ValueError("Q_q must be [B, H, L, d]")
    B, H, L, d = Q_q.shape
    _need(Q_q, torch.int8, "Q_q")
    _need(K_q, torch.int8, "K_q", shape=(B, H, L, d), device=Q_q.device)
    S = _out(S, (B, H, L, L), torch.int32, Q_q.device, "S")
    with _on(Q_q.device):
        _check(lib().intfa_debug_qk(_ptr(Q_q), _ptr(K_q), B, H, L, d, _ptr(S), _stream(stream)), "intfa_debug_qk")
    return S


def intfa_debug_attention_scores(Q_q, K_q, Vt_q, s_Q, s_K, s_V, causal: bool, S, O=None, stream=None):
    """intfa_attention_fwd that also writes the integer logits its softmax
    recovers from the tensor-memory accumulator into S (int32 [B, H, L, L];
    entries the kernel never computes are left as they are)."""
    B, H, L, d = _attn_inputs(Q_q, K_q, Vt_q, s_Q, s_K, s_V)
    _need(S, torch.int32, "S", shape=(B, H, L, L), device=Q_q.device)
    O = _out(O, (B, H, L, d), torch.float16, Q_q.device, "O")
    with _on(Q_q.device):
        _check(lib().intfa_debug_attention_scores(_ptr(Q_q), _ptr(K_q), _ptr(Vt_q), _ptr(s_Q), _ptr(s_K),
                                                  _ptr(s_V), B, H, L, d, int(bool(causal)), _ptr(O), _ptr(S),
                                                  _stream(stream)), "intfa_debug_attention_scores")
    return O


def intfa_debug_wait_timeout(Q_q, K_q, Vt_q, s_Q, s_K, s_V, causal: bool, cap_cycles: int, O=None, stream=None):
    """Launch the attention kernel (d = 64) in its test form that issues no
    copy and no MMA, every wait capped at cap_cycles: each role's wait runs
    out, the kernel records the wait site and returns (read it with
    intfa_device_status)."""
    B, H, L, d = _attn_inputs(Q_q, K_q, Vt_q, s_Q, s_K, s_V)
    O = _out(O, (B, H, L, d), torch.float16, Q_q.device, "O")
    with _on(Q_q.device):
        _check(lib().intfa_debug_wait_timeout(_ptr(Q_q), _ptr(K_q), _ptr(Vt_q), _ptr(s_Q), _ptr(s_K), _ptr(s_V),
                                              B, H, L, d, int(bool(causal)), _ptr(O), int(cap_cycles),
                                              _stream(stream)), "intfa_debug_wait_timeout")
    return O


def intfa_forward_workspace_size(B, H, L, d) -> int:
    return int(lib().intfa_forward_workspace_size(B, H, L, d))


def intfa_forward_host_workspace_size(B, H, L, d) -> int:
    return int(lib().intfa_forward_host_workspace_size(B, H, L, d))


def intfa_forward_workspace_layout(B, H, L, d) -> list[int]:
    """Byte offsets inside intfa_forward's workspace of Q_q, K_q, V_q (int8
    [B, H, L, d] each; V's codes untransposed), s_Q, s_K (fp32 [B, H, L]) and
    s_V (fp32 [B, H])."""
    off = (ctypes.c_size_t * 6)()
    _check(lib().intfa_forward_workspace_layout(B, H, L, d, off), "intfa_forward_workspace_layout")
    return list(off)


def intfa_forward(Q, K, V, causal: bool, O=None, workspace=None, stream=None):
    """fp16 [B, H, L, d] device tensors -> O fp16; quantisation + attention."""
    if not isinstance(Q, torch.Tensor) or Q.dim() != 4:
        raise ValueError("Q must be [B, H, L, d]")
    B, H, L, d = Q.shape
    for t, n in ((Q, "Q"), (K, "K"), (V, "V")):
        _need(t, torch.float16, n, shape=(B, H, L, d), device=Q.device)
    O = _out(O, (B, H, L, d), torch.float16, Q.device, "O")
    workspace = _workspace(workspace, intfa_forward_workspace_size(B, H, L, d), Q.device)
    with _on(Q.device):
        _check(lib().intfa_forward(_ptr(Q), _ptr(K), _ptr(V), B, H, L, d, int(bool(causal)), _ptr(O),
                                   _ptr(workspace), workspace.numel(), _stream(stream)), "intfa_forward")
    return O


def intfa_forward_host(Q_host, K_host, V_host, causal: bool, O_host, workspace, stream=None):
    """Host (pinned) fp16 tensors in and out; copies run inside the call."""
    if not isinstance(Q_host, torch.Tensor) or Q_host.dim() != 4:
        raise ValueError("Q must be [B, H, L, d]")
    B, H, L, d = Q_host.shape
    for t, n in ((Q_host, "Q"), (K_host, "K"), (V_host, "V"), (O_host, "O")):
        if t.is_cuda or t.dtype != torch.float16 or not t.is_contiguous() or tuple(t.shape) != (B, H, L, d):
            raise ValueError(f"{n} must be a contiguous fp16 host tensor of shape {(B, H, L, d)}")
    _need(workspace, torch.uint8, "workspace")
    with _on(workspace.device):
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
