"""Expert parallelism on the GPU: the row-space entry points and
ExpertParallelMoE with the library's kernels.

* G = 1 over a one-rank NCCL group: the expert-parallel path (gather, counts
  exchange, receive plan, expert rows forward/backward, token backward) must
  reproduce the one-GPU layer (MoELayerStep) bit for bit, and the oracle
  within the bf16 tolerance.
* G = 2 and 4 ranks emulated as threads of this process on one GPU (rows
  copied between the ranks' buffers; no kernel waits on another): each
  rank's results against the oracle's one-device layer on all ranks' tokens.
* moe_ep_receive_plan against a brute-force placement, and its data check.
"""
import datetime
import socket

import numpy as np
import pytest
import torch

from mixture_experts_layer_59_b200 import binding as B
from mixture_experts_layer_59_b200 import ep as EP
from mixture_experts_layer_59_b200.layer import MoELayerStep
from oracle import moe_oracle as O

from helpers import BF16_TOL, assert_close, f64

pytestmark = pytest.mark.gpu


def _problem(G, T, d, f, E, k, seed):
    g = torch.Generator().manual_seed(seed)
    bf = lambda *s, sc=1.0: (sc * torch.randn(*s, generator=g)).to(torch.bfloat16)
    x, dout = bf(G * T, d), bf(G * T, d)
    wg = bf(d, E, sc=0.05)
    w1, w3, w2 = bf(E, d, f, sc=0.05), bf(E, d, f, sc=0.05), bf(E, f, d, sc=0.05)
    # routing scores fixed as fp32 values shared by both sides
    lo = torch.randn(G * T, E, generator=g)
    return x, dout, wg, w1, w3, w2, lo


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_ep_one_rank_nccl_is_bit_identical_to_the_layer_and_matches_the_oracle():
    import torch.distributed as dist
    T, d, f, E, k = 640, 256, 256, 8, 2
    x, dout, wg, w1, w3, w2, lo = (t.cuda() for t in _problem(1, T, d, f, E, k, 11))
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        layer = EP.ExpertParallelMoE(EP.TorchDistExchange(), E, k)
        out = layer.forward(x, wg, w1, w3, w2, logits_override=lo)
        g = layer.backward(dout)
        torch.cuda.synchronize()
        B.moe_check_status()
    finally:
        dist.destroy_process_group()
    step = MoELayerStep(T, d, f, E, k, torch.bfloat16, "cuda", B.MOE_ROUND_NONE)
    ref_out = step.forward(x, wg, w1, w3, w2, logits_override=lo)
    ref = step.backward(dout)
    torch.cuda.synchronize()
    B.moe_check_status()
    assert torch.equal(out, ref_out)
    for n in ("dx", "dw1", "dw3", "dw2"):
        assert torch.equal(g[n], ref[n]), n
    for n in ("dw_gate", "dlogits"):
        assert torch.equal(g[n], ref[n]), n
    R = int(step.plan["offsets"][-1])
    assert torch.equal(g["dS"][:R], ref["dS"][:R])
    # and the oracle, on the same fp32 routing scores
    fwd = O.layer_fwd(f64(x), f64(wg), f64(w1), f64(w3), f64(w2), k,
                      logits_override=f64(lo))
    bwd = O.layer_bwd(f64(dout), f64(x), f64(wg), f64(w1), f64(w3), f64(w2), fwd,
                      router_grad_on=False)
    assert_close(out, fwd["out"], "out", BF16_TOL)
    for n in ("dx", "dw1", "dw3", "dw2", "dlogits"):
        assert_close(g[n], bwd[n], n, BF16_TOL)


@pytest.mark.parametrize("G", [2, 4])
def test_ep_emulated_ranks_match_the_oracle(G):
    T, d, f, E, k = 256, 256, 256, 8, 2
    El = E // G
    x, dout, wg, w1, w3, w2, lo = _problem(G, T, d, f, E, k, 20 + G)
    B.lib()
    dev = [t.cuda() for t in (x, dout, wg, w1, w3, w2, lo)]

    def rank_fn(r, ex):
        xc, dc, wgc, w1c, w3c, w2c, loc = dev
        sl, el = slice(r * T, (r + 1) * T), slice(r * El, (r + 1) * El)
        layer = EP.ExpertParallelMoE(ex, E, k)
        out = layer.forward(xc[sl].contiguous(), wgc, w1c[el].contiguous(), w3c[el].contiguous(),
                            w2c[el].contiguous(), logits_override=loc[sl].contiguous())
        g = layer.backward(dc[sl].contiguous())
        torch.cuda.synchronize()
        return dict(out=out.clone(), **{n: g[n].clone() for n in ("dx", "dw1", "dw3", "dw2",
                                                                 "dlogits")})

    res = EP.LocalGroup(G, timeout=120).run(rank_fn)
    B.moe_check_status()
    fwd = O.layer_fwd(f64(x), f64(wg), f64(w1), f64(w3), f64(w2), k, logits_override=f64(lo))
    bwd = O.layer_bwd(f64(dout), f64(x), f64(wg), f64(w1), f64(w3), f64(w2), fwd,
                      router_grad_on=False)
    for r in range(G):
        sl, el = slice(r * T, (r + 1) * T), slice(r * El, (r + 1) * El)
        assert_close(res[r]["out"], fwd["out"][sl], f"out rank {r}", BF16_TOL)
        assert_close(res[r]["dx"], bwd["dx"][sl], f"dx rank {r}", BF16_TOL)
        assert_close(res[r]["dlogits"], bwd["dlogits"][sl], f"dlogits rank {r}", BF16_TOL)
        for n in ("dw1", "dw3", "dw2"):
            assert_close(res[r][n], bwd[n][el], f"{n} rank {r}", BF16_TOL)


def test_ep_receive_plan_matches_brute_force_and_flags_bad_counts():
    rng = np.random.default_rng(4)
    for G, El in [(1, 1), (2, 4), (8, 32), (3, 256)]:
        rows = (rng.integers(0, 5, size=(G, El)) * 128).astype(np.int32)
        lo, rr = B.moe_ep_receive_plan(torch.from_numpy(rows).cuda())
        torch.cuda.synchronize()
        B.moe_check_status()
        want_lo = np.concatenate([[0], np.cumsum(rows.sum(axis=0))])
        want_rr = np.zeros((G, El), np.int64)
        for j in range(El):
            for s in range(G):
                want_rr[s, j] = want_lo[j] + rows[:s, j].sum()
        np.testing.assert_array_equal(lo.cpu().numpy(), want_lo)
        np.testing.assert_array_equal(rr.cpu().numpy(), want_rr)
    # a count that no plan can produce is skipped and reported
    bad = torch.tensor([[128, 7], [256, 128]], dtype=torch.int32).cuda()
    lo, rr = B.moe_ep_receive_plan(bad)
    with pytest.raises(B.MoEError) as ei:
        B.moe_check_status()
    assert ei.value.code == B.MOE_ERR_DEVICE_CHECK and "0x130" in str(ei.value)
    assert lo.cpu().tolist() == [0, 384, 512]
    # dispatch counts are the padded segment lengths of a plan
    logits, idx, gate = B.moe_route(None, None, 2, logits_override=torch.randn(300, 8).cuda(),
                                    T=300, E=8)
    plan = B.moe_permute(idx, gate, logits, 8)
    seg = B.moe_ep_dispatch_counts(plan["offsets"])
    off = plan["offsets"].cpu().numpy()
    np.testing.assert_array_equal(seg.cpu().numpy(), off[1:] - off[:-1])
    B.moe_check_status()


def test_ep_emulated_rank_without_rows():
    """Every token routed to the first rank's experts: the second rank runs
    its grouped GEMMs on an empty row space (offsets all zero) and returns
    zero expert gradients; both ranks match the oracle."""
    G, T, d, f, E, k = 2, 256, 256, 256, 8, 2
    El = E // G
    x, dout, wg, w1, w3, w2, _ = _problem(G, T, d, f, E, k, 31)
    g = torch.Generator().manual_seed(31)
    lo = torch.full((G * T, E), -5.0) + 1e-3 * torch.randn(G * T, E, generator=g)
    lo[:, :El] += 6.0 + torch.rand(G * T, El, generator=g)     # experts 0..El-1: rank 0
    B.lib()
    dev = [t.cuda() for t in (x, dout, wg, w1, w3, w2, lo)]

    def rank_fn(r, ex):
        xc, dc, wgc, w1c, w3c, w2c, loc = dev
        sl, el = slice(r * T, (r + 1) * T), slice(r * El, (r + 1) * El)
        layer = EP.ExpertParallelMoE(ex, E, k)
        out = layer.forward(xc[sl].contiguous(), wgc, w1c[el].contiguous(), w3c[el].contiguous(),
                            w2c[el].contiguous(), logits_override=loc[sl].contiguous())
        gr = layer.backward(dc[sl].contiguous())
        torch.cuda.synchronize()
        return dict(out=out.clone(), rows=layer.routing["local_rows"],
                    **{n: gr[n].clone() for n in ("dx", "dw1", "dw3", "dw2")})

    res = EP.LocalGroup(G, timeout=120).run(rank_fn)
    B.moe_check_status()
    assert res[1]["rows"] == 0
    for n in ("dw1", "dw3", "dw2"):
        assert not bool(res[1][n].any()), n
    fwd = O.layer_fwd(f64(x), f64(wg), f64(w1), f64(w3), f64(w2), k, logits_override=f64(lo))
    bwd = O.layer_bwd(f64(dout), f64(x), f64(wg), f64(w1), f64(w3), f64(w2), fwd,
                      router_grad_on=False)
    for r in range(G):
        sl, el = slice(r * T, (r + 1) * T), slice(r * El, (r + 1) * El)
        assert_close(res[r]["out"], fwd["out"][sl], f"out rank {r}", BF16_TOL)
        assert_close(res[r]["dx"], bwd["dx"][sl], f"dx rank {r}", BF16_TOL)
    assert_close(res[0]["dw1"], bwd["dw1"][:El], "dw1 rank 0", BF16_TOL)
