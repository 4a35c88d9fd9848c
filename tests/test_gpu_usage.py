"""The documented usage: the per-row calls of the binding and the
preallocated step object (with graph capture) give the same results, bit
for bit, on a small layer."""
import pytest
import torch

from mixture_experts_layer_59_b200 import binding as B
from mixture_experts_layer_59_b200 import synth
from mixture_experts_layer_59_b200.layer import MoELayerStep

pytestmark = pytest.mark.gpu


def test_documented_call_sequence_matches_the_step_object():
    cfg = synth.MoEConfig("usage", 300, 256, 256, 8, 2, std=0.05)
    inp = synth.make_inputs(cfg, seed=23, device="cuda")
    x, w_gate, w1, w3, w2, dout = (inp[n] for n in ("x", "w_gate", "w1", "w3", "w2", "dout"))
    T, E, k = cfg.T, cfg.E, cfg.k

    logits, idx, gate = B.moe_route(x, w_gate, k)
    plan = B.moe_permute(idx, gate, logits, E)
    H, Y = B.moe_expert_ffn_fwd(x, w1, w3, w2, plan, k)
    out = B.moe_combine(Y, plan["row_gate"], plan["slot_row"], plan["extra_row"], T, E, k)
    g = B.moe_layer_bwd(dout, x, w_gate, w1, w3, w2, idx, gate, plan, H)
    B.moe_check_status()

    step = MoELayerStep(T, cfg.d, cfg.f, E, k, torch.bfloat16, "cuda", B.MOE_ROUND_NONE)
    out2 = step.forward(x, w_gate, w1, w3, w2).clone()
    grads = {n: t.clone() for n, t in step.backward(dout).items()}
    graph = step.capture(x, w_gate, w1, w3, w2, dout)
    graph.replay()
    torch.cuda.synchronize()
    B.moe_check_status()

    assert torch.isfinite(out.float()).all()
    assert torch.equal(out, out2) and torch.equal(out, step.out)
    for n in ("dx", "dw_gate", "dw1", "dw3", "dw2"):
        assert torch.equal(g[n], grads[n]), n
        assert torch.equal(g[n], step.grads[n]), n


def test_profile_report_counts_every_launch():
    """moe_profile_report lists each kernel with its launch count, total and
    median launch time (the bench's per-kernel rates use the median)."""
    cfg = synth.MoEConfig("usage", 300, 256, 256, 8, 2, std=0.05)
    inp = synth.make_inputs(cfg, seed=29, device="cuda")
    x, w_gate, w1, w3, w2, dout = (inp[n] for n in ("x", "w_gate", "w1", "w3", "w2", "dout"))
    step = MoELayerStep(cfg.T, cfg.d, cfg.f, cfg.E, cfg.k, torch.bfloat16, "cuda",
                        B.MOE_ROUND_NONE)
    B.moe_profile_report()    # forget anything recorded before
    B.moe_profile_enable(True)
    try:
        for _ in range(3):
            step.forward(x, w_gate, w1, w3, w2)
            step.backward(dout)
    finally:
        B.moe_profile_enable(False)
    rep = B.moe_profile_report()
    B.moe_check_status()
    for name in ("tc_router", "perm_count", "tc_up", "tc_down", "tc_dap", "tc_dx", "tc_dw2",
                 "tc_dw13", "token_reduce", "scatter_rows"):
        assert name in rep, name
    for name, (n, total, med) in rep.items():
        assert n % 3 == 0, name           # the same launches in each of the 3 steps
        assert med > 0.0 and total > 0.0, name
        assert med <= total, name         # one launch's time never exceeds the sum
    assert rep["scatter_rows"][0] == 9    # x rows (forward), dO rows and x rows (backward)
    assert B.moe_profile_report() == {}   # the report forgets what it returned
