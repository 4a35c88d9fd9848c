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
