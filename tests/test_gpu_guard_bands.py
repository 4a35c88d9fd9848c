"""Out-of-bounds writes (the race/overflow check that stands in for a
sanitizer here): every output and workspace of one forward + backward is a
view into a larger buffer with guard bands before and after it; the guards
must be untouched afterwards, and the results equal those of an unguarded
run bit for bit."""
import math

import pytest
import torch

from mixture_experts_layer_59_b200 import binding as B
from mixture_experts_layer_59_b200 import synth

pytestmark = pytest.mark.gpu

GUARD = 4096   # elements on each side (a multiple of 16 bytes for every dtype)


class Guarded:
    def __init__(self):
        self.bufs = []

    def __call__(self, shape, dtype):
        n = math.prod(shape)
        buf = torch.empty(GUARD + n + GUARD, dtype=dtype, device="cuda")
        if dtype.is_floating_point:
            buf.normal_()
        elif dtype == torch.uint8:
            buf.random_(0, 256)
        else:
            buf.random_(-(1 << 20), 1 << 20)
        self.bufs.append((buf, n, buf[:GUARD].clone(), buf[GUARD + n:].clone()))
        return buf[GUARD:GUARD + n].view(shape)

    def check(self):
        torch.cuda.synchronize()
        for i, (buf, n, head, tail) in enumerate(self.bufs):
            assert torch.equal(buf[:GUARD], head), f"buffer {i}: write before its start"
            assert torch.equal(buf[GUARD + n:], tail), f"buffer {i}: write past its end"


def _run(inp, cfg, round_mode, g=None):
    x, wg, w1, w3, w2, dout = (inp[n] for n in ("x", "w_gate", "w1", "w3", "w2", "dout"))
    T, d, f, E, k = cfg.T, cfg.d, cfg.f, cfg.E, cfg.k
    cap = B.moe_row_capacity(T, E, k)
    u8 = torch.uint8
    mk = g if g is not None else (lambda shape, dtype: torch.empty(shape, dtype=dtype, device="cuda"))
    logits, idx, gate = B.moe_route(x, wg, k, logit_bias=inp["logit_bias"],
                                    logits=mk((T, E), torch.float32),
                                    idx=mk((T, k), torch.int32), gate=mk((T, k), torch.float32))
    out_plan = {"counts": mk((E,), torch.int32), "offsets": mk((E + 1,), torch.int32),
                "row_token": mk((cap,), torch.int32), "row_gate": mk((cap,), torch.float32),
                "row_slot": mk((cap,), torch.int32), "slot_row": mk((T * k,), torch.int32)}
    if round_mode == B.MOE_ROUND_NEAREST:
        out_plan["extra_row"] = mk((T, E), torch.int32)
    plan = B.moe_permute(idx, gate, logits, E, round_mode, out=out_plan,
                         ws=mk((max(B.moe_permute_workspace_size(T, E, k, round_mode), 1),), u8))
    H, Y = B.moe_expert_ffn_fwd(
        x, w1, w3, w2, plan, k, H=mk((cap, 2 * f), x.dtype), Y_perm=mk((cap, d), x.dtype),
        ws=mk((max(B.moe_ffn_fwd_workspace_size(T, d, f, E, k, B.MOE_BF16), 1),), u8))
    out = B.moe_combine(Y, plan["row_gate"], plan["slot_row"], plan["extra_row"], T, E, k,
                        out=mk((T, d), x.dtype))
    grads = B.moe_layer_bwd(
        dout, x, wg, w1, w3, w2, idx, gate, plan, H,
        out={"dx": mk((T, d), x.dtype), "dw_gate": mk((d, E), torch.float32),
             "dw1": mk((E, d, f), x.dtype), "dw3": mk((E, d, f), x.dtype),
             "dw2": mk((E, f, d), x.dtype), "dS": mk((cap,), torch.float32),
             "dlogits": mk((T, E), torch.float32)},
        ws=mk((max(B.moe_layer_bwd_workspace_size(T, d, f, E, k, B.MOE_BF16), 1),), u8))
    B.moe_check_status()
    torch.cuda.synchronize()
    return dict(logits=logits, idx=idx, gate=gate, H=H, out=out, **grads,
                **{"plan_" + n: t for n, t in plan.items() if t is not None})


@pytest.mark.parametrize("round_mode", [B.MOE_ROUND_NONE, B.MOE_ROUND_NEAREST])
def test_no_write_outside_any_output_or_workspace(round_mode):
    # ragged T, several experts without a full tile, d and f over several N tiles
    cfg = synth.MoEConfig("guard", 1000, 384, 256, 16, 4, std=0.05, routing="zipf")
    inp = synth.make_inputs(cfg, seed=29, device="cuda")
    g = Guarded()
    res = _run(inp, cfg, round_mode, g)
    g.check()
    ref = _run(inp, cfg, round_mode)
    # rows at or past offsets[E] (the padded row count) are never written, and
    # dS exists only for the rows that hold a token
    R = int(ref["plan_offsets"][-1])
    live = ref["plan_row_token"][:R] >= 0
    for n, t in ref.items():
        a = res[n]
        if n in ("H", "plan_row_token", "plan_row_gate", "plan_row_slot"):
            a, t = a[:R], t[:R]
        elif n == "dS":
            a, t = a[:R][live], t[:R][live]
        assert torch.equal(a, t), n
