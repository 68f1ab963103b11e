"""GPU quantisers vs the CPU oracle, bit-exact (codes and fp32 scales)."""
import numpy as np
import pytest
import torch

import oracle
from int8_quantized_attention_token_b200 import intfa
from int8_quantized_attention_token_b200.workloads import WORKLOADS, make_workload

pytestmark = pytest.mark.gpu


def special_rows(d):
    rows = [np.zeros(d), np.full(d, 1e-7)]                   # zero row, fp16 subnormals
    r = np.zeros(d); r[0] = 127.0; r[1:5] = [2.5, -3.5, 0.5, 1.5]; rows.append(r)   # s = 1: ties
    r = np.zeros(d); r[0] = 63.5; r[1:4] = [1.25, -0.75, 0.25]; rows.append(r)     # s = 0.5
    rows.append(np.linspace(-60000, 60000, d))               # near the fp16 maximum
    return np.stack(rows)


@pytest.mark.parametrize("d", [8, 16, 32, 64, 128, 256])
@pytest.mark.parametrize("rows", [1, 7, 1000, 4099])
def test_per_token_bit_exact(rows, d):
    g = torch.Generator().manual_seed(rows * 1000 + d)
    x = (torch.randn(rows, d, generator=g) * torch.rand(rows, 1, generator=g) * 10).half()
    sp = torch.from_numpy(special_rows(d)).half()
    x[: min(rows, sp.shape[0])] = sp[: min(rows, sp.shape[0])]
    q, s = intfa.intfa_quantize_per_token(x.cuda())
    qo, so = oracle.quantize_per_token(x.float().numpy())
    np.testing.assert_array_equal(q.cpu().numpy(), qo)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))


def test_per_token_empty():
    x = torch.empty(0, 64, dtype=torch.float16, device="cuda")
    q, s = intfa.intfa_quantize_per_token(x)
    assert q.numel() == 0 and s.numel() == 0


@pytest.mark.parametrize("transpose", [False, True])
@pytest.mark.parametrize("groups,rows,cols", [(1, 1, 64), (3, 129, 64), (4, 1000, 128), (2, 77, 8),
                                              (5, 4096, 128), (1, 33, 256), (2, 1300, 32),
                                              (3, 2500, 64)])
def test_per_tensor_bit_exact(groups, rows, cols, transpose):
    g = torch.Generator().manual_seed(groups * 7 + rows + cols)
    x = (torch.randn(groups, rows, cols, generator=g) * 3).half()
    x[0, 0, 0] = 0.0
    x[0, -1, -1] = 50.0                                       # the maximum in the last row tile
    if groups > 1:
        x[1] = 0.0                                            # an all-zero group
    q, s = intfa.intfa_quantize_per_tensor(x.cuda(), transpose=transpose)
    qo, so = oracle.quantize_per_tensor(x.float().numpy(), groups)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))
    q = q.cpu().numpy()
    if transpose:
        ld = intfa.intfa_vt_ld(rows)
        assert q.shape == (groups, cols, ld)
        np.testing.assert_array_equal(q[:, :, :rows].transpose(0, 2, 1), qo)
        assert not q[:, :, rows:].any()                       # padding codes are zero
    else:
        np.testing.assert_array_equal(q, qo)


def near_tie_values(amax):
    """Every non-negative finite fp16 x <= amax whose IEEE quotient x / s
    (s = fl32(amax / 127)) lies within 2e-3 of a half-integer, both signs: a
    superset of the elements the kernels' fast rounding leaves to the IEEE
    quotient, and of the exact ties."""
    h = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float32)
    h = h[h <= np.float32(amax)]
    s = np.float32(np.float32(amax) / np.float32(127.0))
    q = h / s
    near = h[np.abs(q - np.floor(q) - np.float32(0.5)) < np.float32(2e-3)]
    assert near.size > 0
    return np.concatenate([near, -near])


@pytest.mark.parametrize("transpose", [False, True])
@pytest.mark.parametrize("amax", [127.0, 100.0, 1.0, 0.0999755859375, 3.0517578125e-05])
def test_per_tensor_near_ties(amax, transpose):
    vals = near_tie_values(amax)
    cols = 128
    rows = max(300, -(-(vals.size + 1) // cols))
    rng = np.random.default_rng(11)
    x = (rng.uniform(-1, 1, (2, rows, cols)) * amax).astype(np.float16).astype(np.float32)
    flat = x[0].reshape(-1)
    flat[-1] = amax                                           # the maximum in the last row tile
    flat[: vals.size] = vals
    x[1] = np.roll(x[0], 77 * cols + 5)
    xh = torch.from_numpy(x).half()
    q, s = intfa.intfa_quantize_per_tensor(xh.cuda(), transpose=transpose)
    qo, so = oracle.quantize_per_tensor(xh.float().numpy(), 2)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))
    q = q.cpu().numpy()
    if transpose:
        q = q[:, :, :rows].transpose(0, 2, 1)
    np.testing.assert_array_equal(q, qo)


@pytest.mark.parametrize("amax", [127.0, 100.0, 0.0999755859375])
def test_per_token_near_ties(amax):
    vals = near_tie_values(amax)
    d = 128
    n = -(-vals.size // (d - 1))
    x = np.zeros((n, d), np.float32)
    x[:, 0] = amax
    body = np.zeros(n * (d - 1), np.float32)
    body[: vals.size] = vals
    x[:, 1:] = body.reshape(n, d - 1)
    xh = torch.from_numpy(x).half()
    q, s = intfa.intfa_quantize_per_token(xh.cuda())
    qo, so = oracle.quantize_per_token(xh.float().numpy())
    np.testing.assert_array_equal(q.cpu().numpy(), qo)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))


@pytest.mark.parametrize("w", [WORKLOADS[2], WORKLOADS[3]], ids=lambda w: w.name)
def test_full_size_quantisation_bit_exact(w):
    Q, K, V = make_workload(w)
    for X in (Q, K):
        q, s = intfa.intfa_quantize_per_token(X.cuda())
        qo, so = oracle.quantize_per_token(X.float().numpy())
        np.testing.assert_array_equal(q.cpu().numpy(), qo)
        np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))
    Vg = V.reshape(w.B * w.H, w.L, w.d)
    q, s = intfa.intfa_quantize_per_tensor(Vg.cuda(), transpose=True)
    qo, so = oracle.quantize_per_tensor(Vg.float().numpy(), w.B * w.H)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))
    np.testing.assert_array_equal(q.cpu().numpy()[:, :, : w.L].transpose(0, 2, 1), qo)


def test_scale_of_every_fp16_magnitude():
    """Rows whose abs-max runs over every finite fp16 magnitude: scales and
    codes equal the oracle's IEEE fp32 results bit for bit."""
    mags = np.arange(1, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float32)
    n = mags.size
    rng = np.random.default_rng(9)
    frac = rng.uniform(-1, 1, (n, 7)).astype(np.float32)
    x = np.concatenate([mags[:, None], (frac * mags[:, None])], axis=1).astype(np.float16)
    xt = torch.from_numpy(x)
    q, s = intfa.intfa_quantize_per_token(xt.cuda())
    qo, so = oracle.quantize_per_token(x.astype(np.float32))
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))
    np.testing.assert_array_equal(q.cpu().numpy(), qo)
    # the same magnitudes as per-tensor abs-maxes
    g = x[:, None, :8].repeat(1, axis=1).reshape(n, 1, 8)
    q2, s2 = intfa.intfa_quantize_per_tensor(torch.from_numpy(np.ascontiguousarray(g)).cuda(), transpose=True)
    qo2, so2 = oracle.quantize_per_tensor(g.astype(np.float32), n)
    np.testing.assert_array_equal(s2.cpu().numpy().view(np.uint32), so2.view(np.uint32))
    np.testing.assert_array_equal(q2.cpu().numpy()[:, :, :1].transpose(0, 2, 1), qo2)


def offset16(x: torch.Tensor) -> torch.Tensor:
    """x's values in a CUDA tensor whose data starts 16 bytes past a 32-byte
    boundary (the quantisers' two-load form; torch allocations are 256-byte
    aligned and take the 32-byte-load form)."""
    flat = torch.empty(x.numel() + 8, dtype=x.dtype, device="cuda")
    y = flat[8:].view(x.shape)
    y.copy_(x.cuda())
    assert y.data_ptr() % 32 == 16
    return y


@pytest.mark.parametrize("d", [16, 64, 128, 256])
def test_per_token_16_byte_aligned_input(d):
    g = torch.Generator().manual_seed(d + 5)
    x = (torch.randn(777, d, generator=g) * 4).half()
    x[3] = 0.0
    q, s = intfa.intfa_quantize_per_token(offset16(x))
    qo, so = oracle.quantize_per_token(x.float().numpy())
    np.testing.assert_array_equal(q.cpu().numpy(), qo)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))


@pytest.mark.parametrize("transpose", [False, True])
@pytest.mark.parametrize("cols", [32, 64, 128])
def test_per_tensor_16_byte_aligned_input(cols, transpose):
    g = torch.Generator().manual_seed(cols + 11)
    rows = 1100
    x = (torch.randn(3, rows, cols, generator=g) * 2).half()
    x[1, -1, 0] = 30.0
    q, s = intfa.intfa_quantize_per_tensor(offset16(x), transpose=transpose)
    qo, so = oracle.quantize_per_tensor(x.float().numpy(), 3)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))
    q = q.cpu().numpy()
    if transpose:
        q = q[:, :, :rows].transpose(0, 2, 1)
    np.testing.assert_array_equal(q, qo)


@pytest.mark.parametrize("groups,rows,cols", [(70, 300, 128), (600, 20, 64), (600, 100, 64)])
def test_per_tensor_many_groups_per_cluster(groups, rows, cols):
    """More groups than the per-head kernel's clusters: each cluster then
    writes one group's codes while reading the next group's abs-max."""
    g = torch.Generator().manual_seed(groups + rows)
    x = (torch.randn(groups, rows, cols, generator=g) * torch.rand(groups, 1, 1, generator=g) * 5).half()
    x[groups // 2] = 0.0
    x[-1, -1, -1] = 60.0
    q, s = intfa.intfa_quantize_per_tensor(x.cuda(), transpose=False)
    qo, so = oracle.quantize_per_tensor(x.float().numpy(), groups)
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))
    np.testing.assert_array_equal(q.cpu().numpy(), qo)
