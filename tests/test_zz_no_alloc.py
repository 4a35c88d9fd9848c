"""The allocation-free permutation entry point (moe_permute_noalloc).

Callers such as plugin hosts that hand over only input and output buffers,
or step loops that must not call cudaMalloc between launches, use this entry
point; its scratch lives in a static device array instead of a workspace.
Its output must equal moe_permute's (round_mode none) exactly, call after
call, even though every call reuses the same static scratch.  The cases
below include the largest the array admits (T = 65536, E = 256, k = 8: every
one of its words is written and read) and an empty call (T = 0), and the
plans are also checked against the CPU oracle's dropless permutation.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from mixture_experts_layer_59_b200 import binding as B
from oracle import moe_oracle as O


def test_noalloc_rejects_oversize_before_touching_the_gpu():
    lib = B.lib()
    fake = ctypes.c_void_p(256)
    rc = lib.moe_permute_noalloc(fake, fake, 65537, 8, 2, 128, fake, fake, fake, fake, fake,
                                 fake, None)
    assert rc == B.MOE_ERR_UNSUPPORTED
    assert b"65536" in lib.moe_last_error()
    rc = lib.moe_permute_noalloc(fake, fake, 100, 257, 2, 128, fake, fake, fake, fake, fake,
                                 fake, None)
    assert rc == B.MOE_ERR_UNSUPPORTED


def _route(T, E, k, seed):
    g = torch.Generator().manual_seed(seed)
    lo = torch.randn(T, E, generator=g).cuda()
    return B.moe_route(None, None, k, logits_override=lo, T=T, E=E)


def _check_equal(got, ref, tag):
    R = int(ref["offsets"][-1].item())
    for name in ("counts", "offsets", "slot_row"):
        assert torch.equal(got[name], ref[name]), (tag, name)
    for name in ("row_token", "row_slot", "row_gate"):
        assert torch.equal(got[name][:R], ref[name][:R]), (tag, name)


def _check_oracle(got, idx, gate, E, tag):
    plan = O.exact_plan(idx.cpu().numpy(), gate.cpu().numpy(), E)
    R = plan["R"]
    i64 = lambda t: t.cpu().numpy().astype(np.int64)
    np.testing.assert_array_equal(i64(got["counts"]), plan["counts"], err_msg=tag)
    np.testing.assert_array_equal(i64(got["offsets"]), plan["offsets"], err_msg=tag)
    np.testing.assert_array_equal(i64(got["row_token"])[:R], plan["row_token"][:R], err_msg=tag)
    np.testing.assert_array_equal(i64(got["row_slot"])[:R], plan["row_slot"][:R], err_msg=tag)
    np.testing.assert_array_equal(i64(got["slot_row"]), plan["slot_row"], err_msg=tag)
    # the row weights are the gates themselves (fp32 values, compared exactly)
    np.testing.assert_array_equal(got["row_gate"][:R].cpu().numpy().astype(np.float64),
                                  plan["row_gate"][:R], err_msg=tag)


@pytest.mark.gpu
def test_noalloc_matches_permute_two_calls_in_a_row():
    # different routings in a row: a call must not see an earlier call's
    # scratch contents; the first case fills the static array to its limit
    cases = [(65536, 256, 8), (5000, 64, 8), (1234, 8, 2), (65536, 256, 8)]
    for call, (T, E, k) in enumerate(cases):
        logits, idx, gate = _route(T, E, k, 100 + call)
        ref = B.moe_permute(idx, gate, logits, E, B.MOE_ROUND_NONE)
        got = B.moe_permute_noalloc(idx, gate, E)
        torch.cuda.synchronize()
        B.moe_check_status()
        _check_equal(got, ref, call)
        if call < 2:
            _check_oracle(got, idx, gate, E, f"call {call}")


@pytest.mark.gpu
def test_noalloc_empty_call_then_full_call():
    E, k = 64, 4
    idx = torch.empty(0, k, dtype=torch.int32, device="cuda")
    gate = torch.empty(0, k, dtype=torch.float32, device="cuda")
    out = dict(counts=torch.full((E,), -7, dtype=torch.int32, device="cuda"),
               offsets=torch.full((E + 1,), -7, dtype=torch.int32, device="cuda"))
    got = B.moe_permute_noalloc(idx, gate, E, out=out)
    ref = B.moe_permute(idx, gate, None, E, B.MOE_ROUND_NONE)
    torch.cuda.synchronize()
    B.moe_check_status()
    assert torch.equal(got["counts"], ref["counts"]) and int(got["counts"].abs().sum()) == 0
    assert torch.equal(got["offsets"], ref["offsets"]) and int(got["offsets"].abs().sum()) == 0
    # and a full call right after the empty one
    logits, idx, gate = _route(3000, E, k, 7)
    ref = B.moe_permute(idx, gate, logits, E, B.MOE_ROUND_NONE)
    got = B.moe_permute_noalloc(idx, gate, E)
    torch.cuda.synchronize()
    B.moe_check_status()
    _check_equal(got, ref, "after empty")
