"""The allocation-free per-tensor quantiser (intfa_quantize_per_tensor_noalloc).

It serves callers that cannot allocate device memory (so cannot pass the
workspace intfa_quantize_per_tensor needs); its scratch is a fixed array
inside the library.  This file is collected last on purpose.  The GPU test
calls the entry point through the C ABI and compares it with the existing
entry point on two calls in a row (the second call must not see the first
call's leftover scratch); the check is bit-exact, as for every quantiser test.
"""
import numpy as np
import pytest
import torch

from int8_quantized_attention_token_b200 import build, intfa

MAX_GROUPS = 4096


def test_rejects_more_groups_than_the_builtin_scratch():
    build.build()
    L = intfa.lib()
    fake = 1 << 20      # never dereferenced: the size check comes first
    assert L.intfa_quantize_per_tensor_noalloc(fake, MAX_GROUPS + 1, 16, 64, 0, fake, fake, None) == 2
    assert L.intfa_quantize_per_tensor_noalloc(fake, 4, 16, 60, 0, fake, fake, None) == 2
    assert L.intfa_quantize_per_tensor_noalloc(None, 0, 16, 64, 0, None, None, None) == 0


@pytest.mark.gpu
@pytest.mark.parametrize("transpose", [False, True])
def test_matches_workspace_entry_point_two_calls(transpose):
    torch.cuda.set_device(0)
    g = torch.Generator().manual_seed(77)
    # first call: large values in many groups; second call: small values and
    # fewer groups, so leftover abs-max scratch from the first would show up
    x1 = (torch.randn(96, 333, 128, generator=g) * 9).half().cuda()
    x2 = (torch.randn(40, 333, 128, generator=g) * 0.01).half().cuda()
    for x in (x1, x2):
        q_ref, s_ref = intfa.intfa_quantize_per_tensor(x, transpose=transpose)
        q, s = intfa.intfa_quantize_per_tensor_noalloc(x, transpose=transpose)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), s_ref.cpu().numpy().view(np.uint32))
        np.testing.assert_array_equal(q.cpu().numpy(), q_ref.cpu().numpy())
    # the largest accepted size still works
    x3 = torch.randn(MAX_GROUPS, 2, 8, generator=g).half().cuda()
    q_ref, s_ref = intfa.intfa_quantize_per_tensor(x3)
    q, s = intfa.intfa_quantize_per_tensor_noalloc(x3)
    torch.cuda.synchronize()
    assert torch.equal(q, q_ref) and torch.equal(s, s_ref)
