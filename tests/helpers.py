"""Shared helpers of the GPU parity tests: run the layer through the C ABI,
run the oracle on the same inputs, and compare with the stated tolerances."""
from __future__ import annotations

import numpy as np
import torch

from mixture_experts_layer_59_b200 import binding as B
from oracle import moe_oracle as O

# Float tolerance for the bf16 path (bf16 storage, fp32 accumulation):
#   max |gpu - ref| <= 1e-2 * max |ref|   and   sum |gpu - ref| / sum |ref| <= 2e-3.
BF16_TOL = (1e-2, 2e-3)
# fp32 path: fp32 storage and accumulation against fp64.
F32_TOL = (1e-4, 1e-5)


def f64(t) -> np.ndarray:
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    return t.detach().to("cpu", torch.float64).numpy()


def i64(t) -> np.ndarray:
    return t.detach().to("cpu", torch.int64).numpy()


def assert_close(gpu, ref, name, tol=BF16_TOL):
    gpu, ref = f64(gpu), f64(ref)
    assert gpu.shape == ref.shape, (name, gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{name}: non-finite values"
    if ref.size == 0:
        return
    diff = np.abs(gpu - ref)
    scale = np.abs(ref).max()
    mx = diff.max() if diff.size else 0.0
    rel = diff.sum() / max(np.abs(ref).sum(), 1e-300)
    if scale == 0:
        assert mx == 0, f"{name}: expected zeros, max |gpu| = {mx}"
        return
    assert mx <= tol[0] * scale, f"{name}: max|d| {mx:.3e} > {tol[0]} * max|ref| {scale:.3e}"
    assert rel <= tol[1], f"{name}: mean relative error {rel:.3e} > {tol[1]}"


def fp32_router_logits(x, w_gate, logit_bias=None):
    """The routing decision input shared by both sides: the oracle's fp64
    logits x W_gate (+bias) rounded once to fp32."""
    lg = f64(x) @ f64(w_gate)
    if logit_bias is not None:
        lg = lg + f64(logit_bias)[None, :]
    return lg.astype(np.float32)


def gpu_layer(inp, k, round_mode, logits32, router_grad=True, dev="cuda", gate_mode=0,
              capacity=-1, noise=None):
    """Forward + backward through the C ABI with the routing logits given."""
    x, wg, w1, w3, w2, dout = (inp[n].to(dev) for n in ("x", "w_gate", "w1", "w3", "w2", "dout"))
    lo = torch.from_numpy(np.ascontiguousarray(logits32)).to(dev)
    T, E = lo.shape
    logits, idx, gate = B.moe_route(x, wg, k, logits_override=lo, gate_mode=gate_mode,
                                    logit_noise=None if noise is None else noise.to(dev))
    plan = B.moe_permute(idx, gate, logits, E, round_mode, gate_mode=gate_mode, capacity=capacity)
    H, Y = B.moe_expert_ffn_fwd(x, w1, w3, w2, plan, k)
    out = B.moe_combine(Y, plan["row_gate"], plan["slot_row"], plan["extra_row"], T, E, k)
    g = B.moe_layer_bwd(dout, x, wg, w1, w3, w2, idx, gate, plan, H, router_grad=router_grad,
                        logits=logits, gate_mode=gate_mode)
    B.moe_check_status()
    torch.cuda.synchronize()
    return dict(logits=logits, idx=idx, gate=gate, plan=plan, H=H, Y=Y, out=out, **g)


def oracle_layer(inp, k, round_mode, logits32, staged=True, router_grad=True, gate_mode=0,
                 capacity=None):
    x, wg, w1, w3, w2, dout = (f64(inp[n]) for n in ("x", "w_gate", "w1", "w3", "w2", "dout"))
    fwd = O.layer_fwd(x, wg, w1, w3, w2, k, round_mode=round_mode,
                      logits_override=np.asarray(logits32, np.float64), staged=staged,
                      gate_mode=gate_mode, capacity=capacity)
    bwd = O.layer_bwd(dout, x, wg, w1, w3, w2, fwd, staged=staged, router_grad_on=router_grad)
    return fwd, bwd


def compare_plan(gp, plan, exact_gate=False):
    """Integer row maps bit-exact; weights to fp32 rounding."""
    R = plan["R"]
    np.testing.assert_array_equal(i64(gp["counts"]), plan["counts"])
    np.testing.assert_array_equal(i64(gp["offsets"]), plan["offsets"])
    np.testing.assert_array_equal(i64(gp["row_token"])[:R], plan["row_token"][:R])
    np.testing.assert_array_equal(i64(gp["row_slot"])[:R], plan["row_slot"][:R])
    np.testing.assert_array_equal(i64(gp["slot_row"]), plan["slot_row"])
    if plan["extra_row"] is not None:
        np.testing.assert_array_equal(i64(gp["extra_row"]), plan["extra_row"])
    np.testing.assert_allclose(f64(gp["row_gate"])[:R], plan["row_gate"][:R], rtol=2e-6, atol=1e-7)


def compare_layer(g, fwd, bwd, tol=BF16_TOL):
    plan = fwd["plan"]
    compare_plan(g["plan"], plan)
    R = plan["R"]
    live = plan["row_token"][:R] >= 0
    assert_close(g["out"], fwd["out"], "out", tol)
    assert_close(f64(g["H"])[:R][live], fwd["H"][:R][live], "H", tol)
    assert_close(f64(g["dS"])[:R][live], bwd["dS"][:R][live], "dS", tol)
    assert_close(g["dlogits"], bwd["dlogits"], "dlogits", tol)
    for n in ("dx", "dw_gate", "dw1", "dw3", "dw2"):
        assert_close(g[n], bwd[n], n, tol)
