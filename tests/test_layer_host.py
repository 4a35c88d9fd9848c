"""Host-side behaviour of the preallocated step object (no GPU: buffers on
the CPU, no kernel launched): argument checks, the row-space capacity, the
capacity-factor conversion and which buffers each routing mode allocates."""
import math

import pytest
import torch

from mixture_experts_layer_59_b200 import binding as B
from mixture_experts_layer_59_b200.layer import MoELayerStep

T, d, f, E, k = 300, 256, 128, 8, 2


def _step(**kw):
    args = dict(dtype=torch.bfloat16, device="cpu", round_mode=B.MOE_ROUND_NONE)
    args.update(kw)
    return MoELayerStep(T, d, f, E, k, **args)


def test_row_space_and_saved_buffers():
    s = _step()
    cap = T * k + E * 128            # every expert segment padded to a 128-row tile
    assert s.cap == cap == B.moe_row_capacity(T, E, k)
    assert tuple(s.H.shape) == (cap, 2 * f) and s.H.dtype == torch.bfloat16
    assert tuple(s.Y.shape) == (cap, d)
    for n in ("row_token", "row_gate", "row_slot"):
        assert tuple(s.plan[n].shape) == (cap,)
    assert tuple(s.plan["slot_row"].shape) == (T * k,)
    assert tuple(s.plan["offsets"].shape) == (E + 1,)
    assert s.plan["extra_row"] is None and s.capacity == -1
    assert tuple(s.grads["dw1"].shape) == (E, d, f) and tuple(s.grads["dw2"].shape) == (E, f, d)
    assert tuple(s.grads["dw_gate"].shape) == (d, E) and s.grads["dw_gate"].dtype == torch.float32


def test_token_rounding_keeps_the_added_row_table():
    s = _step(round_mode=B.MOE_ROUND_NEAREST)
    assert tuple(s.plan["extra_row"].shape) == (T, E)


def test_capacity_factor_becomes_tokens_per_expert():
    s = _step(round_mode=B.MOE_ROUND_CAPACITY, capacity_factor=1.25)
    assert s.capacity == math.ceil(1.25 * T * k / E)
    with pytest.raises(ValueError):
        _step(round_mode=B.MOE_ROUND_CAPACITY)


def test_precision_must_be_known():
    with pytest.raises(ValueError):
        _step(precision="fp16")


def test_mxfp8_step_allocates_quantised_weights():
    s = _step(precision="mxfp8")
    sizes = B.moe_mxfp8_weight_sizes(E, d, f)
    assert [s.wq[n].numel() for n in B.MX_WEIGHT_NAMES] == list(sizes)
    # E4M3 copies of W1|W3 and W2 (one byte per element) and their scale blocks
    assert sizes[0] == E * 2 * f * d and sizes[2] == E * d * f
    assert sizes[1] == E * 2 * f * d // 32 and sizes[3] == E * d * f // 32
