"""The C-ABI library on the host (no GPU needed): it loads, exports every
entry point include/intfa.h declares, and rejects bad arguments before
launching anything."""
import ctypes

import pytest

from int8_quantized_attention_token_b200 import build, intfa


@pytest.fixture(scope="module")
def L():
    build.build()
    return intfa.lib()


def test_exports_every_declared_symbol(L):
    names = intfa.declared_symbols()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for code in range(7):
        assert intfa.status_string(code) not in ("", "unknown status")
    assert intfa.status_string(99) == "unknown status"


def test_vt_ld_and_workspace_sizes(L):
    assert [intfa.intfa_vt_ld(n) for n in (1, 15, 16, 17, 4096)] == [16, 16, 16, 32, 4096]
    assert L.intfa_quantize_per_tensor_workspace_size(128) == 512
    assert L.intfa_quantize_per_tensor_workspace_size(0) == 0
    B, H, Lq, d = 4, 32, 4096, 128
    ws = intfa.intfa_forward_workspace_size(B, H, Lq, d)
    n = B * H * Lq
    assert ws >= 3 * n * d + 2 * 4 * n
    assert intfa.intfa_forward_host_workspace_size(B, H, Lq, d) >= ws + 4 * 2 * n * d
    off = intfa.intfa_forward_workspace_layout(B, H, Lq, d)
    assert off[0] == 0 and all(o % 256 == 0 for o in off) and sorted(off) == off
    assert intfa.intfa_forward_workspace_size(1, 1, 128, 96) == 0


FAKE = 1 << 20   # a 16-byte aligned non-null address; never dereferenced: every call fails its checks


def test_quantize_per_token_rejects(L):
    assert L.intfa_quantize_per_token(None, 0, 64, None, None, None) == 0        # empty: no-op
    assert L.intfa_quantize_per_token(FAKE, -1, 64, FAKE, FAKE, None) == 1
    assert L.intfa_quantize_per_token(None, 4, 64, FAKE, FAKE, None) == 1
    assert L.intfa_quantize_per_token(FAKE, 4, 96, FAKE, FAKE, None) == 2
    assert L.intfa_quantize_per_token(FAKE + 2, 4, 64, FAKE, FAKE, None) == 3
    assert L.intfa_quantize_per_token(FAKE, 4, 64, FAKE + 8, FAKE, None) == 3


def test_quantize_per_tensor_rejects(L):
    ws = L.intfa_quantize_per_tensor_workspace_size(4)
    assert L.intfa_quantize_per_tensor(FAKE, 4, 10, 64, 2, FAKE, FAKE, FAKE, ws, None) == 1
    assert L.intfa_quantize_per_tensor(FAKE, 4, 10, 60, 0, FAKE, FAKE, FAKE, ws, None) == 2
    assert L.intfa_quantize_per_tensor(FAKE, 4, 10, 512, 1, FAKE, FAKE, FAKE, ws, None) == 2
    assert L.intfa_quantize_per_tensor(FAKE, 4, 10, 64, 0, FAKE, FAKE, None, ws, None) == 6
    assert L.intfa_quantize_per_tensor(FAKE, 4, 10, 64, 0, FAKE, FAKE, FAKE, ws - 1, None) == 6
    assert L.intfa_quantize_per_tensor(FAKE + 4, 4, 10, 64, 0, FAKE, FAKE, FAKE, ws, None) == 3
    assert L.intfa_quantize_per_tensor(FAKE, 0, 10, 64, 0, None, None, None, 0, None) == 0


def test_quantize_bits_rejects(L):
    f = L.intfa_quantize_per_token_bits
    assert f(FAKE, 10, 64, 1, FAKE, FAKE, None) == 1      # bits
    assert f(FAKE, 10, 64, 9, FAKE, FAKE, None) == 1
    assert f(FAKE, 10, 96, 4, FAKE, FAKE, None) == 2      # d
    assert f(FAKE + 4, 10, 64, 4, FAKE, FAKE, None) == 3
    assert f(FAKE, 0, 64, 4, None, None, None) == 0


def test_quantize_global_rejects(L):
    ws = L.intfa_quantize_per_tensor_workspace_size(4)
    f = L.intfa_quantize_global
    assert f(FAKE, 4, 10, 12, 0, FAKE, FAKE, FAKE, ws, None) == 2      # cols % 8
    assert f(FAKE, 4, 10, 64, 2, FAKE, FAKE, FAKE, ws, None) == 1      # transpose flag
    assert f(FAKE, 4, 10, 64, 0, FAKE, FAKE, FAKE, ws - 1, None) == 6  # workspace
    assert f(FAKE + 4, 4, 10, 64, 0, FAKE, FAKE, FAKE, ws, None) == 3
    assert f(FAKE, 0, 10, 64, 0, None, None, None, 0, None) == 0       # nothing to do


def test_attention_rejects(L):
    a = [FAKE] * 6
    assert L.intfa_attention_fwd(*a, 1, 1, 128, 96, 0, FAKE, None) == 2           # d
    assert L.intfa_attention_fwd(*a, 0, 1, 128, 64, 0, FAKE, None) == 1           # B
    assert L.intfa_attention_fwd(*a, 1, 1, 0, 64, 0, FAKE, None) == 1             # L
    assert L.intfa_attention_fwd(*a, 1, 1, 128, 64, 2, FAKE, None) == 1           # causal flag
    assert L.intfa_attention_fwd(None, *a[1:], 1, 1, 128, 64, 0, FAKE, None) == 1
    assert L.intfa_attention_fwd(*a, 1, 1, 128, 64, 0, FAKE + 8, None) == 3       # O alignment
    assert L.intfa_attention_fwd(FAKE + 1, *a[1:], 1, 1, 128, 64, 0, FAKE, None) == 3
    assert L.intfa_attention_fwd(*a, 1, 1, 300000, 64, 0, FAKE, None) == 2        # int32 bound
    # fp16-Q variant: Q, K_q, Vt_q, s_K, s_V, B, H, L, d, causal, O, s_Q_out
    q = [FAKE] * 5
    assert L.intfa_attention_fwd_q16(*q, 1, 1, 128, 96, 0, FAKE, None, None) == 2    # d
    assert L.intfa_attention_fwd_q16(*q, 1, 0, 128, 64, 0, FAKE, None, None) == 1    # H
    assert L.intfa_attention_fwd_q16(*q, 1, 1, 128, 64, 3, FAKE, None, None) == 1    # causal flag
    assert L.intfa_attention_fwd_q16(None, *q[1:], 1, 1, 128, 64, 0, FAKE, None, None) == 1
    assert L.intfa_attention_fwd_q16(*q, 1, 1, 128, 64, 0, None, None, None) == 1    # O
    assert L.intfa_attention_fwd_q16(FAKE + 2, *q[1:], 1, 1, 128, 64, 0, FAKE, None, None) == 3
    assert L.intfa_attention_fwd_q16(*q, 1, 1, 128, 64, 0, FAKE, FAKE + 2, None) == 3  # s_Q_out
    assert L.intfa_debug_qk(FAKE, FAKE, 1, 1, 128, 32, FAKE, None) == 2
    assert L.intfa_debug_qk(FAKE, None, 1, 1, 128, 64, FAKE, None) == 1


def test_codesum_attention_rejects(L):
    a = [FAKE] * 6
    f = L.intfa_attention_fwd_codesum
    assert f(*a, 1, 1, 128, 96, 0, FAKE, None) == 2
    assert f(*a, 1, 1, 128, 64, 2, FAKE, None) == 1
    assert f(None, *a[1:], 1, 1, 128, 64, 0, FAKE, None) == 1
    assert f(*a, 1, 1, 128, 64, 0, FAKE + 8, None) == 3


def test_pcodes_attention_rejects(L):
    a = [FAKE] * 6
    f = L.intfa_attention_fwd_pcodes
    assert f(*a, 1, 1, 128, 64, 0, 128, 0, FAKE, None) == 1     # p_levels not 127 / 255
    assert f(*a, 1, 1, 128, 64, 0, 0, 0, FAKE, None) == 1
    assert f(*a, 1, 1, 128, 64, 0, 255, 2, FAKE, None) == 1     # lsum_codes flag
    assert f(*a, 1, 1, 128, 96, 0, 255, 0, FAKE, None) == 2     # d
    assert f(*a, 1, 1, 128, 64, 2, 255, 0, FAKE, None) == 1     # causal flag
    assert f(*a, 1, 1, 128, 64, 0, 255, 0, None, None) == 1     # O
    assert f(None, *a[1:], 1, 1, 128, 64, 0, 255, 0, FAKE, None) == 1
    assert f(FAKE + 4, *a[1:], 1, 1, 128, 64, 0, 255, 0, FAKE, None) == 3


def test_blockscale_attention_rejects(L):
    a = [FAKE] * 6
    f = L.intfa_attention_fwd_blockscale
    assert f(*a, 1, 1, 128, 64, 0, 3, FAKE, None) == 1          # not a power of two
    assert f(*a, 1, 1, 128, 64, 0, 0, FAKE, None) == 1
    assert f(*a, 1, 1, 128, 64, 0, 1 << 17, FAKE, None) == 1
    assert f(*a, 1, 1, 128, 96, 0, 128, FAKE, None) == 2        # d
    assert f(*a, 1, 1, 128, 64, 2, 128, FAKE, None) == 1        # causal flag
    assert f(*a, 1, 1, 128, 64, 0, 128, None, None) == 1        # O
    assert f(FAKE + 4, *a[1:], 1, 1, 128, 64, 0, 128, FAKE, None) == 3


def test_decode_rejects(L):
    ws = L.intfa_decode_workspace_size(1, 2, 128, 4)
    assert ws == 1 * 2 * 4 * 130 * 4
    assert L.intfa_decode_workspace_size(1, 2, 96, 4) == 0
    # q, K_q, s_K, V_q, s_V, B, H, L, d, splits, O, workspace, bytes, stream
    f = L.intfa_decode_fwd
    a = [FAKE] * 5
    assert f(*a, 1, 2, 100, 96, 4, FAKE, FAKE, ws, None) == 2           # d
    assert f(*a, 1, 2, 0, 128, 4, FAKE, FAKE, ws, None) == 1            # L
    assert f(*a, 1, 2, 100, 128, 0, FAKE, FAKE, ws, None) == 1          # splits
    assert f(*a, 1, 2, 100, 128, 4, FAKE, FAKE, ws - 1, None) == 1      # workspace too small
    assert f(*a, 1, 2, 100, 128, 4, FAKE, None, ws, None) == 1
    assert f(FAKE + 8, *a[1:], 1, 2, 100, 128, 4, FAKE, FAKE, ws, None) == 3
    assert f(*a, 1, 2, 100, 128, 4, FAKE + 1, FAKE, ws, None) == 3      # O alignment


def test_index_attention_rejects(L):
    # Q_q, K_q, Vt_q, s_Q, s_K, s_V, B, H, L, d, causal, c, b, O, m_out, l_out, stream
    a = [FAKE] * 6
    f = L.intfa_index_attention_fwd
    assert f(*a, 1, 1, 128, 96, 0, 6.6, 5, FAKE, None, None, None) == 2              # d
    assert f(*a, 1, 1, 65537, 64, 0, 6.6, 5, FAKE, None, None, None) == 2            # int32 bound
    assert f(*a, 0, 1, 128, 64, 0, 6.6, 5, FAKE, None, None, None) == 1              # B
    assert f(*a, 1, 1, 128, 64, 2, 6.6, 5, FAKE, None, None, None) == 1              # causal flag
    assert f(*a, 1, 1, 128, 64, 0, 0.0, 5, FAKE, None, None, None) == 1              # c
    assert f(*a, 1, 1, 128, 64, 0, float("nan"), 5, FAKE, None, None, None) == 1
    assert f(*a, 1, 1, 128, 64, 0, 6.6, 0, FAKE, None, None, None) == 1              # b
    assert f(*a, 1, 1, 128, 64, 0, 6.6, 9, FAKE, None, None, None) == 1
    assert f(*a, 1, 1, 128, 64, 0, 6.6, 5, None, None, None, None) == 1              # O
    assert f(FAKE + 8, *a[1:], 1, 1, 128, 64, 0, 6.6, 5, FAKE, None, None, None) == 3
    assert f(*a, 1, 1, 128, 64, 0, 6.6, 5, FAKE, FAKE + 2, None, None) == 3          # m_out


def test_forward_rejects(L):
    assert L.intfa_forward(FAKE, FAKE, FAKE, 1, 1, 128, 64, 0, FAKE, None, 0, None) == 6
    ws = intfa.intfa_forward_workspace_size(1, 1, 128, 64)
    assert L.intfa_forward(FAKE, FAKE, FAKE, 1, 1, 128, 64, 0, FAKE, FAKE + 16, ws, None) == 3
    assert L.intfa_forward(FAKE, FAKE, FAKE, 1, 1, 128, 80, 0, FAKE, FAKE, ws, None) == 2
    assert L.intfa_forward_host(FAKE, FAKE, FAKE, 1, 1, 128, 64, 0, FAKE, FAKE, ws, None) == 6
    wsh = intfa.intfa_forward_host_workspace_size(1, 1, 128, 64)
    # every check of the host path runs before it touches a stream or the device
    assert L.intfa_forward_host(FAKE, FAKE, FAKE, 1, 1, 128, 64, 2, FAKE, FAKE, wsh, None) == 1   # causal flag
    assert L.intfa_forward_host(None, FAKE, FAKE, 1, 1, 128, 64, 0, FAKE, FAKE, wsh, None) == 1
    assert L.intfa_forward_host(FAKE, FAKE, FAKE, 1, 1, 128, 64, 0, None, FAKE, wsh, None) == 1   # O
    assert L.intfa_forward_host(FAKE, FAKE, FAKE, 1, 1, 128, 64, 0, FAKE, FAKE + 16, wsh, None) == 3
    assert L.intfa_forward_host(FAKE, FAKE, FAKE, 1, 1, 128, 96, 0, FAKE, FAKE, wsh, None) == 2   # d
    assert L.intfa_forward_host(FAKE, FAKE, FAKE, 0, 1, 128, 64, 0, FAKE, FAKE, wsh, None) == 1   # B
    # B H ceil(L / 128) query tiles must fit an int (here 2^24 heads of 1024 tiles)
    assert intfa.intfa_forward_workspace_size(1 << 12, 1 << 12, 131072, 64) == 0
    assert L.intfa_forward(FAKE, FAKE, FAKE, 1 << 12, 1 << 12, 131072, 64, 0, FAKE, FAKE, ws, None) == 2


def test_debug_attention_scores_rejects(L):
    # Q_q, K_q, Vt_q, s_Q, s_K, s_V, B, H, L, d, causal, O, S, stream
    a = [FAKE] * 6
    f = L.intfa_debug_attention_scores
    assert f(*a, 1, 1, 128, 96, 0, FAKE, FAKE, None) == 2              # d
    assert f(*a, 1, 1, 128, 64, 2, FAKE, FAKE, None) == 1              # causal flag
    assert f(*a, 1, 1, 128, 64, 0, FAKE, None, None) == 1              # S
    assert f(*a, 1, 1, 128, 64, 0, None, FAKE, None) == 1              # O
    assert f(*a, 17, 1, 4096, 64, 0, FAKE, FAKE, None) == 2            # B H L L above 2^28
    assert f(*a, 1, 1, 128, 64, 0, FAKE, FAKE + 4, None) == 3          # S alignment


def test_debug_wait_timeout_rejects(L):
    # Q_q, K_q, Vt_q, s_Q, s_K, s_V, B, H, L, d, causal, O, cap_cycles, stream
    a = [FAKE] * 6
    f = L.intfa_debug_wait_timeout
    assert f(*a, 1, 1, 128, 128, 0, FAKE, 20000, None) == 2            # only d = 64 is built
    assert f(*a, 1, 1, 128, 64, 0, FAKE, 999, None) == 1               # cap below 1000
    assert f(*a, 1, 1, 128, 64, 0, FAKE, (1 << 32) + 1, None) == 1     # cap above 2^32
    assert f(*a, 1, 1, 128, 64, 2, FAKE, 20000, None) == 1             # causal flag
    assert f(*a, 1, 1, 128, 64, 0, None, 20000, None) == 1             # O
    assert f(*a, 0, 1, 128, 64, 0, FAKE, 20000, None) == 1             # B
    assert f(FAKE + 4, *a[1:], 1, 1, 128, 64, 0, FAKE, 20000, None) == 3
