"""The fused INT8 attention kernel against the oracle's block-wise online form
(FlashAttention's forward workflow with P codes against the running max),
element by element on small shapes and on sampled rows at full size."""
import numpy as np
import pytest
import torch

from int8_quantized_attention_token_b200 import intfa
from int8_quantized_attention_token_b200.workloads import WORKLOADS, make_qkv, make_workload
from parity import TOL_MAXABS, TOL_MRE, gap, oracle_heads

pytestmark = pytest.mark.gpu


def run_gpu(Q, K, V, causal):
    B, H, L, d = Q.shape
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    Qq, sQ = intfa.intfa_quantize_per_token(Qd)
    Kq, sK = intfa.intfa_quantize_per_token(Kd)
    Vt, sV = intfa.intfa_quantize_per_tensor(Vd.reshape(B * H, L, d), transpose=True)
    O = intfa.intfa_attention_fwd(Qq, Kq, Vt.reshape(B, H, d, -1), sQ, sK, sV.reshape(B, H), causal)
    torch.cuda.synchronize()
    assert intfa.intfa_device_status(clear=True) == 0
    return O.float().cpu().numpy()


def check_all(Q, K, V, causal, report=False):
    B, H, L, d = Q.shape
    O = run_gpu(Q, K, V, causal)
    heads = [(b, h) for b in range(B) for h in range(H)]
    ref = oracle_heads(Q, K, V, causal, heads, two_pass=report, fp64=report)
    got = np.stack([O[b, h] for b, h in heads])
    want = np.stack([ref[k]["O"] for k in heads])
    mx, mre = gap(got, want)
    assert np.isfinite(got).all()
    assert mx <= TOL_MAXABS and mre <= TOL_MRE, (mx, mre)
    if report:
        return {"vs_online": (mx, mre),
                "vs_two_pass": gap(got, np.stack([ref[k]["O2"] for k in heads])),
                "vs_fp64": gap(got, np.stack([ref[k]["Ox"] for k in heads])),
                "oracle_vs_fp64": gap(want, np.stack([ref[k]["Ox"] for k in heads]))}
    return mx, mre


@pytest.mark.parametrize("B,H,L,d,causal", [
    (1, 1, 128, 64, False),          # the 128-token d=64 configuration
    (1, 1, 128, 64, True),
    (1, 2, 256, 128, False),
    (1, 2, 384, 128, True),
    (2, 3, 333, 64, False),          # ragged last block (333 = 2 * 128 + 77)
    (2, 3, 333, 64, True),
    (1, 2, 1000, 128, True),         # ragged, several tiles
    (1, 1, 1, 64, False),            # a single token
    (1, 1, 17, 128, True),
    (1, 1, 130, 128, False),
])
def test_small_shapes(B, H, L, d, causal):
    Q, K, V = make_qkv(B, H, L, d, seed=L + d + causal)
    check_all(Q, K, V, causal)


def test_config_128_d64_seed0():
    """The smallest workload exactly as specified (seed 0), every element."""
    w = WORKLOADS[0]
    Q, K, V = make_workload(w)
    check_all(Q, K, V, w.causal)


def test_config_1024_d64_full():
    w = WORKLOADS[1]
    Q, K, V = make_workload(w)
    r = check_all(Q, K, V, w.causal, report=True)
    print("\n", w.name, r)


@pytest.mark.parametrize("causal", [False, True])
def test_constant_logits_is_mean_of_values(causal):
    B, H, L, d = 1, 2, 300, 128
    _, K, V = make_qkv(B, H, L, d, seed=3)
    Q = torch.zeros_like(K)
    O = run_gpu(Q, K, V, causal)
    ref = oracle_heads(Q, K, V, causal, [(0, 0), (0, 1)])
    for h in range(H):
        mx, mre = gap(O[0, h], ref[(0, h)]["O"])
        assert mx < 2e-3 and mre < 1e-3


def test_outliers_and_large_magnitudes():
    Q, K, V = make_qkv(1, 2, 512, 128, seed=9, outliers=True)
    check_all(Q, K, V, True)
    Q, K, V = make_qkv(1, 2, 512, 64, seed=10, scale=8.0)     # peaky softmax
    check_all(Q, K, V, False)


@pytest.mark.parametrize("w", WORKLOADS[2:], ids=lambda w: w.name)
def test_full_size_sampled_rows(w):
    """The workload at its full size, in the launch the benchmark times; the
    oracle checks sampled rows (first, last and random rows of 3 heads)."""
    Q, K, V = make_workload(w)
    O = run_gpu(Q, K, V, w.causal)
    rng = np.random.default_rng(0)
    heads = [(0, 0), (w.B - 1, w.H - 1), (int(rng.integers(w.B)), int(rng.integers(w.H)))]
    rows = np.unique(np.concatenate([np.arange(0, 3), np.arange(w.L - 3, w.L),
                                     rng.choice(w.L, 40, replace=False)]))
    ref = oracle_heads(Q, K, V, w.causal, heads, rows=rows)
    got = np.stack([O[b, h][rows] for b, h in heads])
    want = np.stack([ref[k]["O"] for k in heads])
    mx, mre = gap(got, want)
    assert mx <= TOL_MAXABS and mre <= TOL_MRE, (mx, mre)


def test_forward_entry_points_match_kernels():
    B, H, L, d = 1, 2, 300, 128
    Q, K, V = make_qkv(B, H, L, d, seed=5)
    O1 = run_gpu(Q, K, V, True)
    O2 = intfa.intfa_forward(Q.cuda(), K.cuda(), V.cuda(), True).float().cpu().numpy()
    np.testing.assert_array_equal(O1, O2)
    ws = torch.empty(intfa.intfa_forward_host_workspace_size(B, H, L, d), dtype=torch.uint8, device="cuda")
    Oh = torch.empty(B, H, L, d, dtype=torch.float16).pin_memory()
    intfa.intfa_forward_host(Q.pin_memory(), K.pin_memory(), V.pin_memory(), True, Oh, ws)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(O1, Oh.float().numpy())


@pytest.mark.parametrize("L,d,causal", [(131072, 64, False), (131072 - 37, 128, True)])
def test_longest_supported_sequence(L, d, causal):
    """The largest L the entry point accepts (and a ragged one just below it):
    1024 query tiles of one head, every key block of a row; sampled rows."""
    Q, K, V = make_qkv(1, 1, L, d, seed=77 + d)
    O = run_gpu(Q, K, V, causal)
    rng = np.random.default_rng(3)
    rows = np.unique(np.concatenate([np.arange(0, 3), np.arange(L - 3, L), rng.choice(L, 10, replace=False)]))
    ref = oracle_heads(Q, K, V, causal, [(0, 0)], rows=rows)
    got = O[0, 0][rows]
    assert np.isfinite(got).all()
    mx, mre = gap(got, ref[(0, 0)]["O"])
    assert mx <= TOL_MAXABS and mre <= TOL_MRE, (mx, mre)


@pytest.mark.parametrize("B,H,L,d,causal", [(2, 5, 4096, 128, True), (1, 6, 8192, 64, False)])
def test_forward_host_chunks_match_device_path(B, H, L, d, causal):
    """intfa_forward_host pipelines its copies over chunks of half the heads
    left, at least 4 (1 MiB of fp16 per head and tensor): 5, 4, 1 and 4, 2
    heads here.  Each chunk is
    its own attention launch, so tiles meet other CTAs and other softmax
    warpgroups than in one launch over all heads; the two warpgroups' shares
    of the row sum then add in another order, which may move O by an fp16 ulp.
    Against intfa_forward: within 1e-3 of max|O| (fp16 rounding level) and in
    the parity bar; two host calls on the same buffers: the same bytes."""
    Q, K, V = make_qkv(B, H, L, d, seed=31 + H)
    Od = intfa.intfa_forward(Q.cuda(), K.cuda(), V.cuda(), causal).float().cpu().numpy()
    ws = torch.empty(intfa.intfa_forward_host_workspace_size(B, H, L, d), dtype=torch.uint8, device="cuda")
    Qp, Kp, Vp = Q.pin_memory(), K.pin_memory(), V.pin_memory()
    outs = []
    for _ in range(2):
        Oh = torch.full((B, H, L, d), float("nan"), dtype=torch.float16).pin_memory()
        intfa.intfa_forward_host(Qp, Kp, Vp, causal, Oh, ws)
        torch.cuda.synchronize()
        assert intfa.intfa_device_status(clear=True) == 0
        outs.append(Oh.clone())
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    Oh = outs[0].float().numpy()
    assert np.isfinite(Oh).all()
    mx, mre = gap(Oh, Od)
    assert mx <= 1e-3 and mre <= 1e-4, (mx, mre)


def schedule_rows(w, nsm=148):
    """Query rows of whole 128-row tiles where the persistent schedule is most
    likely to go wrong, for a causal workload (the kernel's tile order: tiles
    head-major, the heaviest tile of each head first; CTA c takes tiles c,
    c + G, ... with G the largest count <= the SM count coprime to the tiles
    per head; the two softmax warpgroups take alternate key blocks of the
    CTA's stream).  Returns {(b, h): rows}: the first and last query tile of 4
    heads, the last two tiles of CTAs 0 and G - 1, and tiles with an odd and
    an even key-block count (the last block falls to either warpgroup)."""
    ntiles = (w.L + 127) // 128
    total = w.B * w.H * ntiles
    G = nsm
    for cand in range(nsm, nsm // 2, -1):
        if np.gcd(cand, ntiles) == 1:
            G = cand
            break
    tiles = {}

    def add(t):
        bh, tt = divmod(t, ntiles)
        qt = ntiles - 1 - tt            # heaviest first
        tiles.setdefault((bh // w.H, bh % w.H), set()).add(qt)

    for bh in (0, 1, w.B * w.H // 2, w.B * w.H - 1):
        add(bh * ntiles + ntiles - 1)   # query tile 0
        add(bh * ntiles)                # the last query tile
    for c in (0, G - 1):
        for t in list(range(c, total, G))[-2:]:
            add(t)
    add(5 * ntiles + 3)                 # ntiles - 4 key blocks
    add(6 * ntiles + 4)                 # ntiles - 5 key blocks
    return {k: np.concatenate([np.arange(128 * t, min(w.L, 128 * t + 128)) for t in sorted(v)])
            for k, v in tiles.items()}


@pytest.mark.parametrize("w", [WORKLOADS[2], WORKLOADS[4]], ids=lambda w: w.name)
def test_full_size_whole_tiles(w):
    """Every row of the tiles where the persistent schedule is most likely to
    go wrong (first / last tiles of several heads, the last units of the first
    and last CTA, both slots), element by element against the oracle."""
    Q, K, V = make_workload(w)
    O = run_gpu(Q, K, V, w.causal)
    sel = schedule_rows(w)
    for (b, h), rows in sel.items():
        ref = oracle_heads(Q, K, V, w.causal, [(b, h)], rows=rows)
        mx, mre = gap(O[b, h][rows], ref[(b, h)]["O"])
        assert mx <= TOL_MAXABS and mre <= TOL_MRE, ((b, h), mx, mre)
