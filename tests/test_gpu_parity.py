"""GPU parity: the CUDA path through the C ABI against the CPU oracle, element
by element, on seeded inputs that span several tiles and a ragged tail."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_59_b200 import binding as B
from mixture_experts_layer_59_b200 import synth
from oracle import moe_oracle as O

from helpers import (BF16_TOL, F32_TOL, assert_close, compare_layer, compare_plan, f64,
                     fp32_router_logits, gpu_layer, i64, oracle_layer)

pytestmark = pytest.mark.gpu


def _cfg(T, d, f, E, k, dtype="bf16", routing="learned", std=0.05):
    return synth.MoEConfig("test", T, d, f, E, k, dtype=dtype, std=std, routing=routing)


# ------------------------------------------------------------------ routing

def test_route_learned_logits_and_topk():
    cfg = _cfg(1000, 256, 128, 16, 4, std=0.05)
    inp = synth.make_inputs(cfg, seed=3, device="cuda")
    logits, idx, gate = B.moe_route(inp["x"], inp["w_gate"], cfg.k)
    torch.cuda.synchronize()
    ref_logits, ref_idx, _ = O.route(f64(inp["x"]), f64(inp["w_gate"]), cfg.k)
    scale = np.abs(ref_logits).max()
    np.testing.assert_allclose(f64(logits), ref_logits, atol=1e-5 * scale, rtol=0)
    # the top-k set is unique wherever the k-th and (k+1)-th logits are apart
    srt = -np.sort(-ref_logits, axis=1)
    gaps = srt[:, :cfg.k] - srt[:, 1:cfg.k + 1]
    clear = gaps[:, cfg.k - 1] > 1e-4 * scale          # the top-k set is unique
    ordered = np.all(gaps > 1e-4 * scale, axis=1)      # and so is its order
    assert clear.mean() > 0.99
    np.testing.assert_array_equal(np.sort(i64(idx)[clear], 1), np.sort(ref_idx[clear], 1))
    np.testing.assert_array_equal(i64(idx)[ordered], ref_idx[ordered])
    # and the gate is the softmax of the GPU's own top-k logits
    g_ref = O.route(None, None, cfg.k, logits_override=f64(logits))[2]
    np.testing.assert_allclose(f64(gate), g_ref, rtol=1e-6, atol=1e-7)


@pytest.mark.parametrize("T,d,E,k,gate_mode,extras", [
    (1000, 2048, 8, 4, 0, False), (4109, 2048, 8, 2, 1, True), (333, 256, 4, 2, 0, True),
    (77, 512, 5, 5, 1, False), (31, 1024, 8, 8, 0, True), (1, 768, 2, 1, 0, False)])
def test_route_small_e_learned(T, d, E, k, gate_mode, extras):
    """Learned routing with few experts (the tensor-core router at E = 8, the
    generic logits + top-k kernels otherwise), bias, noise and both gate
    modes, ragged T.  Logits against the oracle's fp64 product of the same
    bf16 inputs; choice and gates against the oracle fed the GPU's own
    logits."""
    cfg = _cfg(T, d, 64, E, k, std=0.05)
    inp = synth.make_inputs(cfg, seed=17 + T, device="cuda")
    bias = torch.linspace(-0.2, 0.3, E, device="cuda") if extras else None
    noise = synth.logit_noise(T, E, 0.3, seed=T, device="cuda") if extras else None
    logits, idx, gate = B.moe_route(inp["x"], inp["w_gate"], k, logit_bias=bias,
                                    logit_noise=noise, gate_mode=gate_mode)
    torch.cuda.synchronize()
    ref_l, _, _ = O.route(f64(inp["x"]), f64(inp["w_gate"]), k,
                          logit_bias=None if bias is None else f64(bias),
                          logit_noise=None if noise is None else f64(noise))
    scale = np.abs(ref_l).max()
    np.testing.assert_allclose(f64(logits), ref_l, atol=1e-5 * scale, rtol=0)
    _, ridx, rgate = O.route(None, None, k, logits_override=f64(logits), gate_mode=gate_mode)
    np.testing.assert_array_equal(i64(idx), ridx)
    np.testing.assert_allclose(f64(gate), rgate, rtol=2e-6, atol=1e-7)


@pytest.mark.parametrize("E,k", [(8, 2), (64, 8), (256, 8), (5, 5), (33, 3)])
def test_route_override_ties_bitexact(E, k):
    T = 777
    lo = synth.quantized_logits(T, E, levels=4, seed=E)
    bias = torch.linspace(-0.5, 0.5, E) if E == 33 else None
    logits, idx, gate = B.moe_route(None, None, k, logits_override=lo.cuda(),
                                    logit_bias=None if bias is None else bias.cuda(), T=T, E=E)
    torch.cuda.synchronize()
    ref_l, ref_idx, ref_g = O.route(None, None, k, logits_override=f64(lo),
                                    logit_bias=None if bias is None else f64(bias))
    np.testing.assert_array_equal(i64(idx), ref_idx)
    np.testing.assert_array_equal(f64(logits), f64(torch.from_numpy(ref_l.astype(np.float32))))
    np.testing.assert_allclose(f64(gate), ref_g, rtol=1e-6, atol=1e-7)


# ------------------------------------------------------------------ permutation

@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (255, 8, 2), (1000, 16, 4), (4097, 64, 8),
                                   (3000, 256, 8), (300, 4, 4),
                                   # the block-count scan: several 32-block chunks with a
                                   # ragged tail (few experts), a thread per expert with
                                   # and without a tail of blocks (many experts)
                                   (20000, 8, 4), (70000, 2, 2), (16384, 17, 3), (9000, 32, 8)])
def test_permute_exact_bitexact(T, E, k):
    g = torch.Generator().manual_seed(T + E)
    lo = torch.randn(T, E, generator=g)
    logits, idx, gate = B.moe_route(None, None, k, logits_override=lo.cuda(), T=T, E=E)
    plan_g = B.moe_permute(idx, gate, logits, E, B.MOE_ROUND_NONE)
    torch.cuda.synchronize()
    _, ridx, rgate = O.route(None, None, k, logits_override=f64(lo))
    np.testing.assert_array_equal(i64(idx), ridx)
    compare_plan(plan_g, O.exact_plan(ridx, rgate, E))


@pytest.mark.parametrize("T,E,k,skew", [(1000, 8, 2, 0.0), (1000, 8, 2, 1.5), (5000, 16, 4, 1.1),
                                        (8192, 64, 8, 1.1), (3000, 256, 8, 1.1), (200, 8, 2, 0.0),
                                        (20000, 8, 4, 1.1)])
def test_permute_rounded_bitexact(T, E, k, skew):
    g = torch.Generator().manual_seed(7 * T + E)
    lo = torch.randn(T, E, generator=g)
    if skew:
        rank = torch.randperm(E, generator=g).double() + 1
        lo = lo + (-skew * torch.log(rank)).float()[None, :]
    logits, idx, gate = B.moe_route(None, None, k, logits_override=lo.cuda(), T=T, E=E)
    plan_g = B.moe_permute(idx, gate, logits, E, B.MOE_ROUND_NEAREST)
    torch.cuda.synchronize()
    _, ridx, _ = O.route(None, None, k, logits_override=f64(lo))
    plan = O.rounded_plan(ridx, f64(lo), E)
    assert (plan["dropped"].any() or plan["added"].any()) or T < 256
    compare_plan(plan_g, plan)


# ------------------------------------------------------------------ whole layer

@pytest.mark.parametrize("round_mode", [0, 1])
def test_layer_bf16_small(round_mode):
    """Several M tiles per expert, ragged tails, d and f spanning several N tiles."""
    cfg = _cfg(1000, 256, 256, 8, 2, std=0.05)
    inp = synth.make_inputs(cfg, seed=11, device="cuda")
    lg = fp32_router_logits(inp["x"], inp["w_gate"])
    g = gpu_layer(inp, cfg.k, round_mode, lg)
    fwd, bwd = oracle_layer(inp, cfg.k, round_mode, lg)
    compare_layer(g, fwd, bwd, BF16_TOL)


def test_layer_bf16_many_experts_empty_segments():
    """E=64 with T*k=1536: some experts get no tokens (empty segments, zero dW)."""
    cfg = _cfg(384, 128, 128, 64, 4, std=0.08)
    inp = synth.make_inputs(cfg, seed=5, device="cuda")
    bias = torch.zeros(64)
    bias[40:] = -30.0                     # experts 40..63 are never chosen
    lg = fp32_router_logits(inp["x"], inp["w_gate"], bias)
    g = gpu_layer(inp, cfg.k, 0, lg)
    fwd, bwd = oracle_layer(inp, cfg.k, 0, lg)
    assert (fwd["plan"]["counts"] == 0).sum() >= 24
    compare_layer(g, fwd, bwd, BF16_TOL)
    assert np.all(f64(g["dw1"])[40:] == 0) and np.all(f64(g["dw2"])[40:] == 0)


def test_layer_fp32_tiny_config():
    """The tiny fp32 workload in full (T=256, d=128, f=256, E=8, k=2)."""
    cfg = synth.CONFIGS["tiny_fp32"]
    inp = synth.make_inputs(cfg, seed=0, device="cuda")
    lg = fp32_router_logits(inp["x"], inp["w_gate"])
    g = gpu_layer(inp, cfg.k, 0, lg)
    fwd, bwd = oracle_layer(inp, cfg.k, 0, lg, staged=False)
    compare_layer(g, fwd, bwd, F32_TOL)


def test_layer_router_grad_off_with_override():
    cfg = _cfg(500, 128, 128, 8, 2, routing="uniform")
    inp = synth.make_inputs(cfg, seed=2, device="cuda")
    lg = f64(inp["logits_override"]).astype(np.float32)
    g = gpu_layer(inp, cfg.k, 0, lg, router_grad=False)
    fwd, bwd = oracle_layer(inp, cfg.k, 0, lg, router_grad=False)
    compare_layer(g, fwd, bwd, BF16_TOL)
    assert np.all(f64(g["dw_gate"]) == 0)


def test_zero_tokens_is_a_no_op():
    E, k = 8, 2
    lo = torch.empty(0, E, device="cuda")
    logits, idx, gate = B.moe_route(None, None, k, logits_override=lo, T=0, E=E)
    plan = B.moe_permute(idx, gate, logits, E)
    torch.cuda.synchronize()
    assert i64(plan["offsets"]).tolist() == [0] * (E + 1)
    assert i64(plan["counts"]).tolist() == [0] * E


# ------------------------------------------------------------------ load-balance loss

@pytest.mark.parametrize("T,E,k,skew", [(1000, 8, 2, 0.0), (4097, 64, 8, 1.1), (3000, 256, 8, 1.5)])
def test_balance_loss_and_stats(T, E, k, skew):
    g = torch.Generator().manual_seed(T + E)
    lo = torch.randn(T, E, generator=g)
    if skew:
        rank = torch.randperm(E, generator=g).double() + 1
        lo = lo + (-skew * torch.log(rank)).float()[None, :]
    logits, idx, gate = B.moe_route(None, None, k, logits_override=lo.cuda(), T=T, E=E)
    r = B.moe_balance_loss(idx, gate, E, lam=0.01)
    torch.cuda.synchronize()
    ref = O.balance_loss(i64(idx), f64(gate), E, 0.01)
    st = f64(r["stats"])
    np.testing.assert_allclose(st[0], ref["loss"], rtol=1e-5)
    np.testing.assert_allclose(st[1:], [ref["max_share"], ref["count_cv2"], ref["count_mse"]], rtol=1e-5)
    np.testing.assert_allclose(f64(r["importance"]), ref["importance"], rtol=1e-5, atol=1e-9)
    np.testing.assert_allclose(f64(r["dgate"]), ref["dgate"], rtol=1e-4, atol=1e-9 * np.abs(ref["dgate"]).max())


def test_layer_with_balance_loss_gradient():
    cfg = _cfg(1000, 256, 256, 8, 2, std=0.05)
    inp = synth.make_inputs(cfg, seed=13, device="cuda")
    lg = fp32_router_logits(inp["x"], inp["w_gate"])
    x, wg, w1, w3, w2, dout = (inp[n] for n in ("x", "w_gate", "w1", "w3", "w2", "dout"))
    logits, idx, gate = B.moe_route(x, wg, cfg.k, logits_override=torch.from_numpy(lg).cuda())
    plan = B.moe_permute(idx, gate, logits, cfg.E)
    H, Y = B.moe_expert_ffn_fwd(x, w1, w3, w2, plan, cfg.k)
    bl = B.moe_balance_loss(idx, gate, cfg.E, lam=0.05)
    gr = B.moe_layer_bwd(dout, x, wg, w1, w3, w2, idx, gate, plan, H, gate_grad=bl["dgate"])
    B.moe_check_status()
    torch.cuda.synchronize()
    fwd, _ = oracle_layer(inp, cfg.k, 0, lg)
    rb = O.balance_loss(fwd["idx"], fwd["gate"], cfg.E, 0.05)
    extra = O.gate_grad_to_logits(fwd["idx"], fwd["gate"], rb["dgate"], cfg.E)
    bwd = O.layer_bwd(f64(dout), f64(x), f64(wg), f64(w1), f64(w3), f64(w2), fwd, extra_dlogits=extra)
    for n in ("dlogits", "dw_gate", "dx", "dw1"):
        assert_close(gr[n], bwd[n], n, BF16_TOL)


# ------------------------------------------------------------------ routing variants

@pytest.mark.parametrize("E,k", [(8, 2), (64, 8), (256, 8), (33, 3)])
def test_route_softmax_then_topk_gates(E, k):
    """Gates = softmax over all E logits, the k largest kept; same expert choice."""
    T = 777
    lo = synth.quantized_logits(T, E, levels=4, seed=E + 1)
    logits, idx, gate = B.moe_route(None, None, k, logits_override=lo.cuda(), T=T, E=E,
                                    gate_mode=B.MOE_GATE_SOFTMAX_TOPK)
    torch.cuda.synchronize()
    _, ref_idx, ref_g = O.route(None, None, k, logits_override=f64(lo), gate_mode=1)
    np.testing.assert_array_equal(i64(idx), ref_idx)
    np.testing.assert_allclose(f64(gate), ref_g, rtol=2e-6, atol=1e-7)
    assert np.all(f64(gate).sum(1) <= 1 + 1e-6)


def test_route_softmax_then_topk_tensor_core_router():
    """The tensor-core router epilogue's normaliser over all E logits."""
    cfg = _cfg(1000, 256, 128, 64, 8, std=0.05)
    inp = synth.make_inputs(cfg, seed=4, device="cuda")
    bias = torch.linspace(-0.3, 0.3, cfg.E, device="cuda")
    logits, idx, gate = B.moe_route(inp["x"], inp["w_gate"], cfg.k, logit_bias=bias,
                                    gate_mode=B.MOE_GATE_SOFTMAX_TOPK)
    torch.cuda.synchronize()
    # gates against the oracle fed the GPU's own logits and choice
    lg = f64(logits)
    p = np.exp(lg - lg.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    np.testing.assert_allclose(f64(gate), np.take_along_axis(p, i64(idx), 1), rtol=2e-6, atol=1e-7)
    _, ref_idx, _ = O.route(None, None, cfg.k, logits_override=lg, gate_mode=1)
    np.testing.assert_array_equal(i64(idx), ref_idx)


@pytest.mark.parametrize("T,E,k,skew,gate_mode,cf", [
    (1000, 8, 2, 1.5, 0, 1.0), (1000, 8, 2, 1.5, 1, 1.25), (5000, 16, 4, 1.1, 0, 1.0),
    (8192, 64, 8, 1.1, 1, 1.0), (3000, 256, 8, 1.1, 0, 2.0), (200, 8, 2, 0.0, 0, 0.0),
    (300, 4, 4, 0.0, 1, 1.0)])
def test_permute_capacity_bitexact(T, E, k, skew, gate_mode, cf):
    """Capacity-factor dropping: every row map bit-exact (cf 0 drops every pair)."""
    g = torch.Generator().manual_seed(5 * T + E)
    lo = torch.randn(T, E, generator=g)
    if skew:
        rank = torch.randperm(E, generator=g).double() + 1
        lo = lo + (-skew * torch.log(rank)).float()[None, :]
    cap = B.capacity_from_factor(T, E, k, cf)
    logits, idx, gate = B.moe_route(None, None, k, logits_override=lo.cuda(), T=T, E=E,
                                    gate_mode=gate_mode)
    plan_g = B.moe_permute(idx, gate, logits, E, B.MOE_ROUND_CAPACITY, gate_mode=gate_mode,
                           capacity=cap)
    torch.cuda.synchronize()
    _, ridx, rgate = O.route(None, None, k, logits_override=f64(lo), gate_mode=gate_mode)
    plan = O.make_plan(ridx, rgate, f64(lo), E, round_mode=2, gate_mode=gate_mode, capacity=cap)
    assert plan_g["extra_row"] is None
    if skew and cf <= 1.0:                 # uneven load: the busiest experts drop
        assert plan["dropped"].any()
    compare_plan(plan_g, plan)


@pytest.mark.parametrize("T,E,k,skew", [(1000, 8, 2, 1.5), (8192, 64, 8, 1.1), (3000, 256, 8, 1.1)])
def test_permute_rounded_softmax_then_topk_bitexact(T, E, k, skew):
    """Token rounding with scores from the softmax over all E logits."""
    g = torch.Generator().manual_seed(11 * T + E)
    lo = torch.randn(T, E, generator=g)
    rank = torch.randperm(E, generator=g).double() + 1
    lo = lo + (-skew * torch.log(rank)).float()[None, :]
    logits, idx, gate = B.moe_route(None, None, k, logits_override=lo.cuda(), T=T, E=E,
                                    gate_mode=1)
    plan_g = B.moe_permute(idx, gate, logits, E, B.MOE_ROUND_NEAREST, gate_mode=1)
    torch.cuda.synchronize()
    _, ridx, rgate = O.route(None, None, k, logits_override=f64(lo), gate_mode=1)
    plan = O.make_plan(ridx, rgate, f64(lo), E, round_mode=1, gate_mode=1)
    assert plan["added"].any() or plan["dropped"].any()
    compare_plan(plan_g, plan)


@pytest.mark.parametrize("round_mode,gate_mode,cf", [(0, 1, None), (1, 1, None), (2, 0, 1.0),
                                                    (2, 1, 1.25), (2, 0, 0.0)])
def test_layer_bf16_routing_variants(round_mode, gate_mode, cf):
    """The whole layer under each routing variant, against the oracle."""
    cfg = _cfg(1000, 256, 256, 8, 2, std=0.05)
    inp = synth.make_inputs(cfg, seed=17, device="cuda")
    bias = torch.tensor([0.6, 0.4, 0.2, 0.0, 0.0, -0.2, -0.4, -0.6])   # uneven load
    lg = fp32_router_logits(inp["x"], inp["w_gate"], bias)
    cap = B.capacity_from_factor(cfg.T, cfg.E, cfg.k, cf) if round_mode == 2 else -1
    g = gpu_layer(inp, cfg.k, round_mode, lg, gate_mode=gate_mode, capacity=cap)
    fwd, bwd = oracle_layer(inp, cfg.k, round_mode, lg, gate_mode=gate_mode,
                            capacity=cap if round_mode == 2 else None)
    if round_mode == 2:
        assert fwd["plan"]["dropped"].any()
    compare_layer(g, fwd, bwd, BF16_TOL)


def test_layer_softmax_then_topk_with_balance_loss_gradient():
    cfg = _cfg(1000, 256, 256, 8, 2, std=0.05)
    inp = synth.make_inputs(cfg, seed=19, device="cuda")
    lg = fp32_router_logits(inp["x"], inp["w_gate"])
    x, wg, w1, w3, w2, dout = (inp[n] for n in ("x", "w_gate", "w1", "w3", "w2", "dout"))
    logits, idx, gate = B.moe_route(x, wg, cfg.k, logits_override=torch.from_numpy(lg).cuda(),
                                    gate_mode=1)
    plan = B.moe_permute(idx, gate, logits, cfg.E)
    H, Y = B.moe_expert_ffn_fwd(x, w1, w3, w2, plan, cfg.k)
    bl = B.moe_balance_loss(idx, gate, cfg.E, lam=0.05)
    gr = B.moe_layer_bwd(dout, x, wg, w1, w3, w2, idx, gate, plan, H, gate_grad=bl["dgate"],
                         logits=logits, gate_mode=1)
    B.moe_check_status()
    torch.cuda.synchronize()
    fwd, _ = oracle_layer(inp, cfg.k, 0, lg, gate_mode=1)
    rb = O.balance_loss(fwd["idx"], fwd["gate"], cfg.E, 0.05)
    extra = O.gate_grad_to_logits(fwd["idx"], fwd["gate"], rb["dgate"], cfg.E, gate_mode=1,
                                  logits=fwd["logits"])
    bwd = O.layer_bwd(f64(dout), f64(x), f64(wg), f64(w1), f64(w3), f64(w2), fwd, extra_dlogits=extra)
    for n in ("dlogits", "dw_gate", "dx", "dw1"):
        assert_close(gr[n], bwd[n], n, BF16_TOL)


# ------------------------------------------------------------------ noisy top-k gating

@pytest.mark.parametrize("E,k,gate_mode", [(8, 2, 0), (64, 8, 1), (256, 8, 0)])
def test_route_noisy_scores_bitexact(E, k, gate_mode):
    """Routing noise is added after the bias in fp32; the oracle routes the
    same fp32 scores."""
    T = 999
    lo = torch.randn(T, E, generator=torch.Generator().manual_seed(E))
    bias = torch.linspace(-0.5, 0.5, E)
    eps = synth.logit_noise(T, E, 1.0, seed=E)
    logits, idx, gate = B.moe_route(None, None, k, logits_override=lo.cuda(), logit_bias=bias.cuda(),
                                    T=T, E=E, gate_mode=gate_mode, logit_noise=eps.cuda())
    torch.cuda.synchronize()
    scores = (lo + bias[None, :]) + eps                     # the same two fp32 adds
    _, ref_idx, ref_g = O.route(None, None, k, logits_override=f64(scores), gate_mode=gate_mode)
    np.testing.assert_array_equal(f64(logits), f64(scores))
    np.testing.assert_array_equal(i64(idx), ref_idx)
    np.testing.assert_allclose(f64(gate), ref_g, rtol=2e-6, atol=1e-7)
    clean = O.route(None, None, k, logits_override=f64(lo + bias[None, :]))[1]
    assert (i64(idx) != clean).any()                       # the noise changed some choices


@pytest.mark.parametrize("gate_mode", [0, 1])
def test_route_noisy_tensor_core_router(gate_mode):
    cfg = _cfg(1000, 256, 128, 64, 8, std=0.05)
    inp = synth.make_inputs(cfg, seed=8, device="cuda")
    eps = synth.logit_noise(cfg.T, cfg.E, 0.5, seed=8, device="cuda")
    logits, idx, gate = B.moe_route(inp["x"], inp["w_gate"], cfg.k, gate_mode=gate_mode,
                                    logit_noise=eps)
    torch.cuda.synchronize()
    ref = f64(inp["x"]) @ f64(inp["w_gate"]) + f64(eps)
    scale = np.abs(ref).max()
    np.testing.assert_allclose(f64(logits), ref, atol=1e-5 * scale, rtol=0)
    # the choice and gates follow the GPU's own noisy scores exactly
    _, own_idx, own_g = O.route(None, None, cfg.k, logits_override=f64(logits), gate_mode=gate_mode)
    np.testing.assert_array_equal(i64(idx), own_idx)
    np.testing.assert_allclose(f64(gate), own_g, rtol=2e-6, atol=1e-7)


@pytest.mark.parametrize("round_mode,gate_mode", [(0, 0), (1, 1)])
def test_layer_noisy_routing(round_mode, gate_mode):
    cfg = _cfg(1000, 256, 256, 8, 2, std=0.05)
    inp = synth.make_inputs(cfg, seed=23, device="cuda")
    lg = fp32_router_logits(inp["x"], inp["w_gate"])
    eps = synth.logit_noise(cfg.T, cfg.E, 0.02, seed=23)
    g = gpu_layer(inp, cfg.k, round_mode, lg, gate_mode=gate_mode, noise=eps)
    noisy32 = (torch.from_numpy(lg) + eps).numpy()          # the scores the GPU routed on
    fwd, bwd = oracle_layer(inp, cfg.k, round_mode, noisy32, gate_mode=gate_mode)
    compare_layer(g, fwd, bwd, BF16_TOL)


@pytest.mark.parametrize("d,E,k,round_mode", [(384, 32, 4, 1), (128, 16, 2, 1), (640, 24, 8, 0),
                                              (896, 8, 3, 1)])
def test_layer_bf16_fused_dx_shapes(d, E, k, round_mode):
    """Shapes of the fused dx pass (E <= 32) whose row width is not a multiple
    of 32 vectors, with rows added by rounding, and k of every size class."""
    cfg = _cfg(700, d, 128, E, k, std=0.05)
    inp = synth.make_inputs(cfg, seed=d + E, device="cuda")
    bias = torch.linspace(1.0, -1.0, E)                 # uneven load: rounding adds rows
    lg = fp32_router_logits(inp["x"], inp["w_gate"], bias)
    g = gpu_layer(inp, cfg.k, round_mode, lg)
    fwd, bwd = oracle_layer(inp, cfg.k, round_mode, lg)
    if round_mode:
        assert fwd["plan"]["added"].any()
    compare_layer(g, fwd, bwd, BF16_TOL)


# ------------------------------------------------------------------ degenerate shapes

@pytest.mark.parametrize("T,E,k,round_mode", [
    (300, 8, 1, 0),       # top-1 routing: every token has one row, gates are 1
    (260, 4, 4, 0),       # k = E: every token goes to every expert
    (260, 4, 4, 1),       # ... with token rounding (counts 260 -> 256: drops only)
    (1, 8, 2, 0),         # a single token
    (129, 16, 8, 1),      # one more token than a tile, maximal k
])
def test_layer_degenerate_routing_shapes(T, E, k, round_mode):
    cfg = _cfg(T, 128, 128, E, k, std=0.08)
    inp = synth.make_inputs(cfg, seed=T + E + k, device="cuda")
    lg = fp32_router_logits(inp["x"], inp["w_gate"])
    g = gpu_layer(inp, cfg.k, round_mode, lg)
    fwd, bwd = oracle_layer(inp, cfg.k, round_mode, lg)
    if k == 1:
        assert np.all(fwd["gate"] == 1.0)
    if k == E:
        assert np.all(np.sort(fwd["idx"], 1) == np.arange(E))
    compare_layer(g, fwd, bwd, BF16_TOL)


@pytest.mark.parametrize("T,E,k", [(300, 8, 1), (1, 8, 2)])
def test_mxfp8_degenerate_routing_shapes(T, E, k):
    cfg = _cfg(T, 256, 256, E, k, std=0.05)
    inp = synth.make_inputs(cfg, seed=7 * T + k, device="cuda")
    x, wg, w1, w3, w2, dout = (inp[n] for n in ("x", "w_gate", "w1", "w3", "w2", "dout"))
    lg = fp32_router_logits(x, wg)
    logits, idx, gate = B.moe_route(x, wg, k, logits_override=torch.from_numpy(lg).cuda())
    plan = B.moe_permute(idx, gate, logits, E)
    wq = B.moe_mxfp8_quantize_weights(w1, w3, w2)
    H, Y = B.moe_expert_ffn_fwd_mxfp8(x, wq, plan, k, E, cfg.f)
    out = B.moe_combine(Y, plan["row_gate"], plan["slot_row"], plan["extra_row"], T, E, k)
    torch.cuda.synchronize()
    fwd = O.layer_fwd(f64(x), f64(wg), f64(w1), f64(w3), f64(w2), k,
                      logits_override=lg.astype(np.float64), precision="mxfp8")
    assert_close(out, fwd["out"], "out", BF16_TOL)


def test_device_check_reports_and_clears():
    """Failure detection without a GPU fault: expert ids out of range are
    flagged by the permutation kernels (device status word, code 0x120) and
    skipped; moe_check_status reports the flag once, then it is clear, and the
    valid slots are still placed."""
    T, E, k = 500, 8, 2
    g = torch.Generator().manual_seed(41)
    lo = torch.randn(T, E, generator=g)
    logits, idx, gate = B.moe_route(None, None, k, logits_override=lo.cuda(), T=T, E=E)
    torch.cuda.synchronize()
    bad = idx.clone()
    bad[3, 0] = E          # one past the last expert
    bad[77, 1] = -3
    plan = B.moe_permute(bad, gate, logits, E, B.MOE_ROUND_NONE)
    with pytest.raises(B.MoEError) as ei:
        B.moe_check_status()
    assert ei.value.code == B.MOE_ERR_DEVICE_CHECK and "0x120" in str(ei.value)
    B.moe_check_status()   # cleared by the read
    slot_row = i64(plan["slot_row"]).reshape(T, k)
    assert slot_row[3, 0] == -1 and slot_row[77, 1] == -1
    valid = i64(bad) >= 0
    valid &= i64(bad) < E
    assert (slot_row[valid] >= 0).all()
    assert int(i64(plan["counts"]).sum()) == int(valid.sum())


def test_bounded_wait_expires_then_next_call_is_clean():
    """Failure detection of the bounded device waits, without a GPU fault: the
    test hook makes the next tensor-core GEMM's producer issue no copies, so
    the MMA issuer's wait for a full stage runs out (5 ms limit) with nothing
    in flight; the kernel records a 0x2nn code, frees its TMEM and returns.
    moe_check_status reports MOE_ERR_DEVICE_TIMEOUT once, and the same call
    repeated afterwards gives bit-identical results to a clean run."""
    T, d, f, E, k = 512, 256, 256, 8, 2
    g = torch.Generator().manual_seed(43)
    x = (torch.randn(T, d, generator=g)).to(torch.bfloat16).cuda()
    w1, w3 = ((0.05 * torch.randn(E, d, f, generator=g)).to(torch.bfloat16).cuda() for _ in range(2))
    w2 = (0.05 * torch.randn(E, f, d, generator=g)).to(torch.bfloat16).cuda()
    lo = torch.randn(T, E, generator=g).cuda()
    logits, idx, gate = B.moe_route(None, None, k, logits_override=lo, T=T, E=E)
    plan = B.moe_permute(idx, gate, logits, E)
    H0, Y0 = B.moe_expert_ffn_fwd(x, w1, w3, w2, plan, k)
    B.moe_check_status()
    assert B.lib().moe_debug_expire_next_wait(5_000_000) == 0
    B.moe_expert_ffn_fwd(x, w1, w3, w2, plan, k)
    with pytest.raises(B.MoEError) as ei:
        B.moe_check_status()
    assert ei.value.code == B.MOE_ERR_DEVICE_TIMEOUT and "0x20" in str(ei.value)
    B.moe_check_status()   # cleared by the read
    H1, Y1 = B.moe_expert_ffn_fwd(x, w1, w3, w2, plan, k)
    B.moe_check_status()
    R = int(plan["offsets"][-1].item())
    assert torch.equal(H1[:R], H0[:R]) and torch.equal(Y1[:R], Y0[:R])
    # a cancelled request leaves the next launch alone
    assert B.lib().moe_debug_expire_next_wait(5_000_000) == 0
    assert B.lib().moe_debug_expire_next_wait(0) == 0
    H2, _ = B.moe_expert_ffn_fwd(x, w1, w3, w2, plan, k)
    B.moe_check_status()
    assert torch.equal(H2[:R], H0[:R])


@pytest.mark.parametrize("T,d,E,k,round_mode,shift", [(1000, 2048, 8, 4, B.MOE_ROUND_NONE, 0),
                                                     (777, 7168, 16, 2, B.MOE_ROUND_NEAREST, 0),
                                                     (130, 128, 4, 1, B.MOE_ROUND_NONE, 0),
                                                     (0, 256, 8, 2, B.MOE_ROUND_NONE, 0),
                                                     # rows that are not 32-byte multiples, and
                                                     # a destination 16 but not 32 bytes aligned:
                                                     # the 16-byte kernel
                                                     (300, 8, 8, 2, B.MOE_ROUND_NONE, 0),
                                                     (257, 24, 4, 3, B.MOE_ROUND_NEAREST, 0),
                                                     (500, 256, 8, 4, B.MOE_ROUND_NONE, 8)])
def test_gather_rows_bit_exact_with_padding_zeroed(T, d, E, k, round_mode, shift):
    """moe_gather_rows (the row gather behind every grouped GEMM): row r of
    the row space is row row_token[r] of the token-major source, bit for bit,
    including rows added by token rounding; padding rows are zeros, and rows
    at or beyond offsets[E] are left untouched."""
    g = torch.Generator().manual_seed(T + d)
    x = torch.randn(max(T, 1), d, generator=g).to(torch.bfloat16)[:T].cuda()
    lo = torch.randn(T, E, generator=g).cuda()
    logits, idx, gate = B.moe_route(None, None, k, logits_override=lo, T=T, E=E)
    plan = B.moe_permute(idx, gate, logits, E, round_mode)
    cap = B.moe_row_capacity(T, E, k)
    # sentinel-filled destination, starting `shift` elements into its buffer
    flat = torch.full((shift + cap * d,), 7.0, dtype=torch.bfloat16, device="cuda")
    out = flat[shift:].view(cap, d)
    assert out.data_ptr() % 16 == 0
    B.moe_gather_rows(x, plan, k, out=out)
    torch.cuda.synchronize()
    B.moe_check_status()
    R = int(plan["offsets"][-1])
    tok = plan["row_token"][:R].long()
    live = tok >= 0
    want = torch.zeros(R, d, dtype=torch.bfloat16, device="cuda")
    want[live] = x[tok[live]]
    assert torch.equal(out[:R], want)
    assert bool((out[R:] == 7.0).all())
