"""The fused attention with V_hat read in its natural [B, H, L, d] layout (the
P V product takes the V_hat tile N-major) against the transposed-V form and
the oracle: the INT32 P V products are exact either way, so the two GPU
outputs must agree bit for bit on the same codes, and the per-head V codes of
both quantiser layouts must be each other's transpose."""
import numpy as np
import pytest
import torch

from int8_quantized_attention_token_b200 import intfa
from int8_quantized_attention_token_b200.workloads import WORKLOADS, make_qkv, make_workload
from parity import TOL_MAXABS, TOL_MRE, gap, oracle_heads

pytestmark = pytest.mark.gpu


def both_layouts(Q, K, V, causal):
    B, H, L, d = Q.shape
    Qq, sQ = intfa.intfa_quantize_per_token(Q.cuda())
    Kq, sK = intfa.intfa_quantize_per_token(K.cuda())
    Vd = V.cuda().reshape(B * H, L, d)
    Vt, sVt = intfa.intfa_quantize_per_tensor(Vd, transpose=True)
    Vr, sVr = intfa.intfa_quantize_per_tensor(Vd, transpose=False)
    assert torch.equal(sVt.view(torch.int32), sVr.view(torch.int32))
    assert torch.equal(Vt[:, :, :L].transpose(1, 2), Vr)
    Ot = intfa.intfa_attention_fwd(Qq, Kq, Vt.reshape(B, H, d, -1), sQ, sK, sVt.reshape(B, H), causal)
    Or = intfa.intfa_attention_fwd_vrows(Qq, Kq, Vr.reshape(B, H, L, d), sQ, sK, sVr.reshape(B, H), causal)
    torch.cuda.synchronize()
    assert intfa.intfa_device_status(clear=True) == 0
    return Ot, Or


@pytest.mark.parametrize("B,H,L,d,causal", [
    (1, 1, 1, 64, False),
    (1, 1, 17, 128, True),
    (1, 2, 128, 64, True),
    (2, 3, 333, 64, False),
    (2, 3, 333, 128, True),
    (1, 2, 1000, 128, True),
    (1, 1, 640, 64, True),
])
def test_vrows_bit_identical_and_oracle(B, H, L, d, causal):
    Q, K, V = make_qkv(B, H, L, d, seed=7 * L + d + causal)
    Ot, Or = both_layouts(Q, K, V, causal)
    assert torch.equal(Ot.view(torch.int16), Or.view(torch.int16))
    heads = [(b, h) for b in range(B) for h in range(H)]
    ref = oracle_heads(Q, K, V, causal, heads)
    O = Or.float().cpu().numpy()
    mx, mre = gap(np.stack([O[b, h] for b, h in heads]), np.stack([ref[k]["O"] for k in heads]))
    assert mx <= TOL_MAXABS and mre <= TOL_MRE, (mx, mre)


@pytest.mark.parametrize("w", [WORKLOADS[2], WORKLOADS[4]], ids=lambda w: w.name)
def test_vrows_bit_identical_full_size(w):
    Q, K, V = make_workload(w)
    Ot, Or = both_layouts(Q, K, V, w.causal)
    assert torch.equal(Ot.view(torch.int16), Or.view(torch.int16))


def test_forward_workspace_holds_the_codes():
    """After intfa_forward, its workspace holds the quantisers' outputs at the
    offsets intfa_forward_workspace_layout reports: Q_q, K_q, V_q (V's codes
    untransposed) and the three scale arrays, equal to the standalone calls."""
    B, H, L, d = 2, 3, 333, 128
    Q, K, V = [t.cuda() for t in make_qkv(B, H, L, d, seed=5)]
    ws = torch.empty(intfa.intfa_forward_workspace_size(B, H, L, d), dtype=torch.uint8, device="cuda")
    intfa.intfa_forward(Q, K, V, True, workspace=ws)
    torch.cuda.synchronize()
    assert intfa.intfa_device_status(clear=True) == 0
    off = intfa.intfa_forward_workspace_layout(B, H, L, d)
    n = B * H * L * d

    def view(i, count, dtype):
        nbytes = count * torch.tensor([], dtype=dtype).element_size()
        return ws[off[i]:off[i] + nbytes].view(dtype)

    Qq, sQ = intfa.intfa_quantize_per_token(Q)
    Kq, sK = intfa.intfa_quantize_per_token(K)
    Vq, sV = intfa.intfa_quantize_per_tensor(V.reshape(B * H, L, d), transpose=False)
    assert torch.equal(view(0, n, torch.int8), Qq.reshape(-1))
    assert torch.equal(view(1, n, torch.int8), Kq.reshape(-1))
    assert torch.equal(view(2, n, torch.int8), Vq.reshape(-1))
    assert torch.equal(view(3, B * H * L, torch.float32).view(torch.int32), sQ.reshape(-1).view(torch.int32))
    assert torch.equal(view(4, B * H * L, torch.float32).view(torch.int32), sK.reshape(-1).view(torch.int32))
    assert torch.equal(view(5, B * H, torch.float32).view(torch.int32), sV.reshape(-1).view(torch.int32))


def test_forward_captured_in_a_cuda_graph():
    """intfa_forward (with V's quantiser forked onto the library's side stream)
    captured into a CUDA graph and replayed gives the eager call's bytes."""
    B, H, L, d = 1, 4, 640, 128
    Q, K, V = [t.cuda() for t in make_qkv(B, H, L, d, seed=9)]
    ws = torch.empty(intfa.intfa_forward_workspace_size(B, H, L, d), dtype=torch.uint8, device="cuda")
    O_eager = intfa.intfa_forward(Q, K, V, True, workspace=ws)   # first call: makes the side stream
    torch.cuda.synchronize()
    O = torch.empty_like(O_eager)
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s, capture_error_mode="thread_local"):
            intfa.intfa_forward(Q, K, V, True, O=O, workspace=ws, stream=s)
    for _ in range(3):
        O.zero_()
        g.replay()
    torch.cuda.synchronize()
    assert intfa.intfa_device_status(clear=True) == 0
    assert torch.equal(O.view(torch.int16), O_eager.view(torch.int16))
