"""The whole layer step (route, permute, expert FFN, combine, backward) runs
inside one CUDA graph: every entry point only enqueues work on the caller's
stream.  A replayed graph must reproduce the eager step bit for bit, also
after the inputs change in place."""
import pytest
import torch

from mixture_experts_layer_59_b200 import binding as B
from mixture_experts_layer_59_b200 import synth
from mixture_experts_layer_59_b200.layer import MoELayerStep

pytestmark = pytest.mark.gpu


def _outputs(step):
    g = step.grads
    R = int(step.plan["offsets"][-1])            # rows past R are never written
    return [step.out.clone(), step.H[:R].clone(), step.idx.clone(), step.plan["offsets"].clone(),
            g["dx"].clone(), g["dw_gate"].clone(), g["dw1"].clone(), g["dw3"].clone(),
            g["dw2"].clone(), g["dlogits"].clone()]


@pytest.mark.parametrize("round_mode,precision", [(0, "bf16"), (1, "bf16"), (0, "mxfp8")])
def test_captured_step_matches_eager(round_mode, precision):
    cfg = synth.MoEConfig("test", 2000, 256, 256, 8, 2, std=0.05)
    inp = synth.make_inputs(cfg, seed=31, device="cuda")
    x, wg, w1, w3, w2, dout = (inp[n] for n in ("x", "w_gate", "w1", "w3", "w2", "dout"))
    eager = MoELayerStep(cfg.T, cfg.d, cfg.f, cfg.E, cfg.k, round_mode=round_mode,
                         precision=precision, balance_lambda=0.01)
    graphed = MoELayerStep(cfg.T, cfg.d, cfg.f, cfg.E, cfg.k, round_mode=round_mode,
                           precision=precision, balance_lambda=0.01)
    graph = graphed.capture(x, wg, w1, w3, w2, dout)
    for trial in range(2):
        if trial:                                   # new inputs, same buffers
            x.copy_(torch.randn_like(x))
            dout.copy_(torch.randn_like(dout))
        eager.forward(x, wg, w1, w3, w2)
        eager.backward(dout)
        graph.replay()
        torch.cuda.synchronize()
        B.moe_check_status()
        for a, b in zip(_outputs(eager), _outputs(graphed)):
            assert torch.equal(a, b)
