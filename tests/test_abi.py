"""Host-side checks of the C ABI: the library loads, exports every entry point
that include/moe.h declares, sizes workspaces consistently, and rejects bad
arguments before launching anything (no GPU needed)."""
import ctypes
import os
import re

import pytest

from mixture_experts_layer_59_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_0-9]+\s*\*?\s*(moe_[a-z_0-9]+)\s*\(", src, re.M)
    return names


def test_library_exports_every_declared_symbol():
    lib = B.lib()
    names = _declared()
    assert "moe_route" in names and "moe_layer_bwd" in names
    for n in names:
        assert hasattr(lib, n), n
    assert set(B.EXPORTS) >= set(names)


def test_version_and_capacity():
    assert B.moe_version() >= 10000
    assert B.moe_row_capacity(16384, 8, 4) == 16384 * 4 + 8 * 128


def test_workspace_sizes_monotone():
    a = B.moe_layer_bwd_workspace_size(1000, 256, 256, 8, 2, B.MOE_BF16)
    b = B.moe_layer_bwd_workspace_size(2000, 256, 256, 8, 2, B.MOE_BF16)
    assert 0 < a < b
    assert B.moe_permute_workspace_size(100, 8, 2, 1) > B.moe_permute_workspace_size(100, 8, 2, 0)
    assert B.moe_ffn_fwd_workspace_size(100, 256, 256, 8, 2, B.MOE_F32) > 0


def _rc_route(**kw):
    args = dict(x=None, wg=None, T=4, d=128, E=8, k=2, dtype=B.MOE_BF16, gm=0, lo=None, lb=None,
                ln=None, logits=None, idx=None, gate=None, stream=None)
    args.update(kw)
    lib = B.lib()
    return lib.moe_route(args["x"], args["wg"], args["T"], args["d"], args["E"], args["k"],
                         args["dtype"], args["gm"], args["lo"], args["lb"], args["ln"],
                         args["logits"],
                         args["idx"],
                         args["gate"], args["stream"])


@pytest.mark.parametrize("kw,code", [
    (dict(k=0), -2), (dict(k=9), -2), (dict(E=1, k=2), -2), (dict(E=300), -2),
    (dict(dtype=7), -2), (dict(T=-1), -1), (dict(gm=2), -1),
])
def test_route_rejects_bad_shapes(kw, code):
    assert _rc_route(**kw) == code
    assert len(B.lib().moe_last_error()) > 0


def test_route_rejects_null_outputs():
    assert _rc_route() == -1
    assert b"NULL" in B.lib().moe_last_error()


def test_permute_rejects_tile_and_mode():
    lib = B.lib()
    fake = ctypes.c_void_p(16)
    rc = lib.moe_permute(fake, fake, fake, 4, 8, 2, 0, 64, 0, -1, fake, fake, fake, fake, fake, fake,
                         None, fake, 1 << 20, None)
    assert rc == -2
    rc = lib.moe_permute(fake, fake, fake, 4, 8, 2, 3, 128, 0, -1, fake, fake, fake, fake, fake, fake,
                         None, fake, 1 << 20, None)
    assert rc == -1
    # rounding needs logits and extra_row
    rc = lib.moe_permute(fake, fake, None, 4, 8, 2, 1, 128, 0, -1, fake, fake, fake, fake, fake, fake,
                         None, fake, 1 << 20, None)
    assert rc == -1
    # capacity mode: a capacity is required, extra_row is not
    rc = lib.moe_permute(fake, fake, fake, 4, 8, 2, 2, 128, 0, -1, fake, fake, fake, fake, fake,
                         fake, None, fake, 1 << 20, None)
    assert rc == -1 and b"capacity" in lib.moe_last_error()
    # gate_mode out of range
    rc = lib.moe_permute(fake, fake, fake, 4, 8, 2, 1, 128, 5, -1, fake, fake, fake, fake, fake,
                         fake, fake, fake, 1 << 20, None)
    assert rc == -1 and b"gate_mode" in lib.moe_last_error()
    # workspace too small
    rc = lib.moe_permute(fake, fake, fake, 4, 8, 2, 0, 128, 0, -1, fake, fake, fake, fake, fake, fake,
                         None, fake, 8, None)
    assert rc == -5


def test_ffn_rejects_unaligned_dims_and_small_workspace():
    lib = B.lib()
    fake = ctypes.c_void_p(256)
    rc = lib.moe_expert_ffn_fwd(fake, fake, fake, fake, fake, fake, fake, None, 16, 100, 128, 8, 2,
                                B.MOE_BF16, fake, fake, fake, 1 << 30, None)
    assert rc == -2
    rc = lib.moe_expert_ffn_fwd(fake, fake, fake, fake, fake, fake, fake, None, 16, 128, 128, 8, 2,
                                B.MOE_BF16, fake, fake, fake, 16, None)
    assert rc == -5
    odd = ctypes.c_void_p(258)
    rc = lib.moe_expert_ffn_fwd(odd, fake, fake, fake, fake, fake, fake, None, 16, 128, 128, 8, 2,
                                B.MOE_BF16, fake, fake, fake, 1 << 30, None)
    assert rc == -1


def test_bwd_rejects_missing_w_gate_with_router_grad():
    lib = B.lib()
    f = ctypes.c_void_p(256)
    args = [f, f, None, f, f, f, f, f, None, None, 0, f, f, f, f, None, f, 16, 128, 128, 8, 2,
            B.MOE_BF16, 1, f, f, f, f, f, None, None, f, 1 << 40, None]
    assert lib.moe_layer_bwd(*args) == -1
    assert b"w_gate" in lib.moe_last_error()


def test_bwd_softmax_topk_gates_need_logits():
    lib = B.lib()
    f = ctypes.c_void_p(256)
    args = [f, f, f, f, f, f, f, f, None, None, B.MOE_GATE_SOFTMAX_TOPK, f, f, f, f, None, f, 16,
            128, 128, 8, 2, B.MOE_BF16, 1, f, f, f, f, f, None, None, f, 1 << 40, None]
    assert lib.moe_layer_bwd(*args) == -1
    assert b"logits" in lib.moe_last_error()


def test_ffn_requires_slot_row():
    lib = B.lib()
    fake = ctypes.c_void_p(256)
    rc = lib.moe_expert_ffn_fwd(fake, fake, fake, fake, fake, fake, None, None, 16, 128, 128, 8, 2,
                                B.MOE_BF16, fake, fake, fake, 1 << 30, None)
    assert rc == -1 and b"slot_row" in lib.moe_last_error()


def test_balance_loss_rejects_empty_batch_and_small_workspace():
    lib = B.lib()
    f = ctypes.c_void_p(256)
    assert lib.moe_balance_loss(f, f, 0, 8, 2, 0.1, f, f, None, f, 1 << 20, None) == -1
    assert lib.moe_balance_loss(f, f, 100, 8, 2, 0.1, f, f, None, f, 4, None) == -5


def test_mxfp8_entry_points_check_their_arguments():
    lib = B.lib()
    f = ctypes.c_void_p(256)
    sizes = (ctypes.c_size_t * 8)()
    assert lib.moe_mxfp8_weight_sizes(8, 2048, 1024, sizes) == 0
    n = 8 * 2048 * 1024
    assert list(sizes) == [2 * n, 2 * n // 32, n, n // 32, n, n // 32, n, n // 32]
    assert lib.moe_mxfp8_weight_sizes(8, 2000, 1024, sizes) == -2       # d % 128 != 0
    # the four backward outputs are all given or all NULL
    rc = lib.moe_mxfp8_quantize_weights(f, f, f, 8, 256, 256, f, f, f, f, f, None, f, f, None)
    assert rc == -1 and b"all set or all NULL" in lib.moe_last_error()
    # forward: workspace too small is refused before any launch
    rc = lib.moe_expert_ffn_fwd_mxfp8(f, f, f, f, f, f, f, f, None, 16, 256, 256, 8, 2, f, f, f,
                                      16, None)
    assert rc == -5
    assert B.moe_ffn_fwd_mxfp8_workspace_size(16, 256, 256, 8, 2) > 0
    # backward: the quantised weights are required
    args = [f, f, f, f, f, f, None, f, f, f, f, f, None, None, 0, f, f, f, f, None, f, 16, 256,
            256, 8, 2, 1, 0, f, f, f, f, f, None, None, f, 1 << 40, None]
    assert lib.moe_layer_bwd_mxfp8(*args) == -1 and b"w1rq" in lib.moe_last_error()
    assert (B.moe_layer_bwd_mxfp8_workspace_size(16, 256, 256, 8, 2)
            > B.moe_layer_bwd_workspace_size(16, 256, 256, 8, 2, B.MOE_BF16))
    # MXFP8 weight gradients: four more quantised row-space operands
    assert (B.moe_layer_bwd_mxfp8_workspace_size(16, 256, 256, 8, 2, wgrad=True)
            > B.moe_layer_bwd_mxfp8_workspace_size(16, 256, 256, 8, 2))
    args[6:10] = [f, f, f, f]
    args[27] = 2
    assert lib.moe_layer_bwd_mxfp8(*args) == -1 and b"wgrad_mxfp8" in lib.moe_last_error()
    args[27], args[22] = 1, 384          # d not a multiple of 256
    assert lib.moe_layer_bwd_mxfp8(*args) == -2 and b"256" in lib.moe_last_error()
