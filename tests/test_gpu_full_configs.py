"""GPU parity at the full workload sizes (coarse, pool, fine, sparse, and
sparse with token rounding), in the launch configuration bench.py times.

The oracle cannot run whole layers of this size in float64 in seconds, so it
checks what it can compute one by one, exactly:
  * the routing plan (counts, offsets, every row map) in full, bit-exact;
  * out, dx, dlogits and dS of sampled tokens (each depends only on the token
    and its experts' weights);
  * sampled columns of dW1/dW3 and rows of dW2 for the most and least loaded
    experts and one more;
  * dW_gate through the property dW_gate = x^T dlogits, which holds at any size.
Expert weights are copied to the host one expert at a time.
"""
import numpy as np
import pytest
import torch

from mixture_experts_layer_59_b200 import binding as B
from mixture_experts_layer_59_b200 import synth
from oracle import moe_oracle as O

from helpers import (BF16_TOL, assert_close, compare_plan, f64, fp32_router_logits, gpu_layer,
                     i64)

pytestmark = pytest.mark.gpu


class DeviceExperts:
    """fp64 host copy of expert e of an [E, a, b] device tensor, on demand."""

    def __init__(self, t, keep=16):
        self.t, self.keep, self.cache = t, keep, {}

    def __getitem__(self, e):
        e = int(e)
        if e not in self.cache:
            if len(self.cache) >= self.keep:
                self.cache.pop(next(iter(self.cache)))
            self.cache[e] = self.t[e].to("cpu", torch.float64).numpy()
        return self.cache[e]


# (workload, routing, round_mode, sampled tokens, gate_mode, capacity factor)
CASES = [
    ("coarse", "learned", 0, 64, 0, None),
    ("coarse", "uniform", 0, 64, 0, None),
    ("pool", "uniform", 0, 64, 0, None),
    ("pool", "gauss", 0, 64, 0, None),
    ("fine", "learned", 0, 64, 0, None),
    ("sparse", "zipf", 0, 12, 0, None),
    ("sparse", "zipf", 1, 12, 0, None),
    ("coarse", "learned", 2, 64, 1, 1.0),     # softmax over all E, capacity factor 1
    ("fine", "learned", 1, 64, 1, None),      # softmax over all E, token rounding
    ("sparse", "zipf", 2, 12, 0, 1.25),
]


@pytest.mark.parametrize("name,routing,round_mode,n_tok,gate_mode,cf", CASES,
                         ids=[f"{c[0]}-{c[1]}-round{c[2]}-gate{c[4]}" for c in CASES])
def test_full_size_layer(name, routing, round_mode, n_tok, gate_mode, cf):
    cfg = synth.CONFIGS[name].with_(routing=routing)
    T, d, f, E, k = cfg.T, cfg.d, cfg.f, cfg.E, cfg.k
    cap = B.capacity_from_factor(T, E, k, cf) if round_mode == 2 else -1
    inp = synth.make_inputs(cfg, seed=0, device="cuda")
    router_grad = inp["logits_override"] is None
    x64, wg64 = f64(inp["x"]), f64(inp["w_gate"])
    if router_grad:
        logits32 = fp32_router_logits(x64, wg64, inp["logit_bias"])
        # the tensor-core router itself, against the oracle's logits
        lg, idx_g, gate_g = B.moe_route(inp["x"], inp["w_gate"], k, logit_bias=inp["logit_bias"],
                                        gate_mode=gate_mode)
        torch.cuda.synchronize()
        lg = f64(lg)
        scale = np.abs(logits32).max()
        assert np.abs(lg - logits32).max() <= 1e-5 * scale
        srt = -np.sort(-logits32.astype(np.float64), axis=1)
        gaps = srt[:, :k] - srt[:, 1:k + 1]
        clear = gaps[:, k - 1] > 1e-4 * scale          # top-k set is unique
        ordered = np.all(gaps > 1e-4 * scale, axis=1)  # and so is its order
        ref_idx = O.route(None, None, k, logits_override=logits32.astype(np.float64))[1]
        np.testing.assert_array_equal(np.sort(i64(idx_g)[clear], 1), np.sort(ref_idx[clear], 1))
        np.testing.assert_array_equal(i64(idx_g)[ordered], ref_idx[ordered])
        # top-k flips against the fp64 logits: tokens whose chosen expert set
        # differs.  Every flip must sit at a near-tie (the k-th and (k+1)-th
        # fp64 logits within the router's rounding); the count is reported.
        l64 = x64 @ wg64 + (f64(inp["logit_bias"])[None, :] if inp["logit_bias"] is not None
                            else 0.0)
        set64 = np.sort(O.route(None, None, k, logits_override=l64)[1], 1)
        flip = np.any(np.sort(i64(idx_g), 1) != set64, axis=1)
        s64 = -np.sort(-l64, axis=1)
        margin = s64[:, k - 1] - s64[:, k]
        mag = np.maximum(np.abs(s64[:, k - 1]), np.abs(s64[:, k]))
        assert np.all(margin[flip] <= 1e-4 * scale), margin[flip].max()
        near = margin <= 1e-5 * mag
        print(f"\ntop-k flips [{name}/{routing}/gate{gate_mode}]: {int(flip.sum())} of {T} tokens "
              f"differ from the fp64 top-k set; {int((flip & near).sum())} of them, and "
              f"{int(near.sum())} tokens in all, have a k-th margin <= 1e-5 |l|; largest flip "
              f"margin {float(margin[flip].max()) if flip.any() else 0.0:.3g} (logit scale "
              f"{scale:.3g})")
        # gates: the oracle's gate rule applied to the GPU's own logits and choice
        g_ref = O.route(None, None, k, logits_override=lg, gate_mode=gate_mode)[2]
        same = np.all(i64(idx_g) == O.route(None, None, k, logits_override=lg)[1], axis=1)
        np.testing.assert_allclose(f64(gate_g)[same], g_ref[same], rtol=5e-6, atol=1e-7)
        del lg, idx_g, gate_g
    else:
        logits32 = f64(inp["logits_override"]).astype(np.float32)

    g = gpu_layer(inp, k, round_mode, logits32, router_grad=router_grad, gate_mode=gate_mode,
                  capacity=cap)

    # routing plan, in full
    lg64 = logits32.astype(np.float64)
    _, idx, gate = O.route(None, None, k, logits_override=lg64, gate_mode=gate_mode)
    plan = O.make_plan(idx, gate, lg64, E, round_mode=round_mode, gate_mode=gate_mode,
                       capacity=cap if round_mode == 2 else None)
    np.testing.assert_array_equal(i64(g["idx"]), idx)
    compare_plan(g["plan"], plan)
    if round_mode == 1:
        assert plan["R"] < O.exact_plan(idx, gate, E)["R"]   # rounding removed padding rows
    if round_mode == 2:
        assert plan["dropped"].any()
    fwd = dict(logits=lg64, idx=idx, gate=gate, plan=plan)

    W1, W3, W2 = DeviceExperts(inp["w1"]), DeviceExperts(inp["w3"]), DeviceExperts(inp["w2"])
    dout64 = f64(inp["dout"])
    rng = np.random.default_rng(1234)
    tokens = sorted(set([0, T - 1] + list(rng.choice(T, n_tok - 2, replace=False))))
    s = O.sampled_tokens(tokens, dout64, x64, wg64, W1, W3, W2, fwd, router_grad_on=router_grad)
    out_g, dx_g, dl_g = f64(g["out"]), f64(g["dx"]), f64(g["dlogits"])
    assert_close(out_g[tokens], np.stack([s["out"][t] for t in tokens]), "out", BF16_TOL)
    assert_close(dx_g[tokens], np.stack([s["dx"][t] for t in tokens]), "dx", BF16_TOL)
    assert_close(dl_g[tokens], np.stack([s["dlogits"][t] for t in tokens]), "dlogits", BF16_TOL)
    rows = sorted(s["dS"])
    assert_close(f64(g["dS"])[rows], np.array([s["dS"][r] for r in rows]), "dS", BF16_TOL)

    # weight gradients: sampled columns of the most / least loaded and one more expert
    counts = np.diff(plan["offsets"])
    live = np.nonzero(counts > 0)[0]
    experts = sorted({int(live[np.argmax(counts[live])]), int(live[np.argmin(counts[live])]),
                      int(rng.choice(live))})
    cols = sorted(rng.choice(f, 16, replace=False))
    dw1, dw3, dw2 = g["dw1"], g["dw3"], g["dw2"]
    for e in experts:
        ref = O.expert_grad_slices(e, cols, dout64, x64, W1[e], W3[e], W2[e], fwd)
        assert_close(f64(dw1[e][:, cols]), ref["dw1"], f"dw1[{e}]", BF16_TOL)
        assert_close(f64(dw3[e][:, cols]), ref["dw3"], f"dw3[{e}]", BF16_TOL)
        assert_close(f64(dw2[e][cols, :]), ref["dw2"], f"dw2[{e}]", BF16_TOL)
    empty = np.nonzero(counts == 0)[0]
    if len(empty):
        e0 = int(empty[0])
        assert float(dw1[e0].abs().max()) == 0.0 and float(dw2[e0].abs().max()) == 0.0

    # dW_gate = x^T dlogits (property at any size), or zero without a router gradient
    if router_grad:
        assert_close(g["dw_gate"], x64.T @ dl_g, "dw_gate", BF16_TOL)
    else:
        assert float(g["dw_gate"].abs().max()) == 0.0
