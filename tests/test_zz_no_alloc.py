"""The allocation-free permutation entry point (moe_permute_noalloc).

Callers such as plugin hosts that hand over only input and output buffers,
or step loops that must not call cudaMalloc between launches, use this entry
point; its scratch lives in a static device array instead of a workspace.
Its output must equal moe_permute's (round_mode none) exactly, call after
call, even though every call reuses the same static scratch.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from mixture_experts_layer_59_b200 import binding as B


def test_noalloc_rejects_oversize_before_touching_the_gpu():
    lib = B.lib()
    fake = ctypes.c_void_p(256)
    rc = lib.moe_permute_noalloc(fake, fake, 65537, 8, 2, 128, fake, fake, fake, fake, fake,
                                 fake, None)
    assert rc == -2
    assert b"65536" in lib.moe_last_error()


@pytest.mark.gpu
def test_noalloc_matches_permute_two_calls_in_a_row():
    # two different routings in a row: the second call must not see the
    # first call's scratch contents
    for call, (T, E, k) in enumerate([(5000, 64, 8), (1234, 8, 2)]):
        g = torch.Generator().manual_seed(100 + call)
        lo = torch.randn(T, E, generator=g).cuda()
        logits, idx, gate = B.moe_route(None, None, k, logits_override=lo, T=T, E=E)
        ref = B.moe_permute(idx, gate, logits, E, B.MOE_ROUND_NONE)
        got = B.moe_permute_noalloc(idx, gate, E)
        torch.cuda.synchronize()
        B.moe_check_status()
        R = int(ref["offsets"][-1].item())
        for name in ("counts", "offsets", "slot_row"):
            assert torch.equal(got[name], ref[name]), (call, name)
        for name in ("row_token", "row_slot", "row_gate"):
            assert torch.equal(got[name][:R], ref[name][:R]), (call, name)
        # the row weights are the gates themselves (fp32, bit-exact)
        np.testing.assert_array_equal(got["row_gate"][:R].cpu().numpy(),
                                      ref["row_gate"][:R].cpu().numpy())
