"""GPU parity of the MXFP8 expert forward against the oracle's MXFP8
definition (OCP MX, E4M3 elements, E8M0 scale per 32 along K).

Quantised codes and scales that both sides compute from the same bf16 inputs
(weights, token rows) are compared bit for bit; A is quantised from each
side's own SwiGLU output, so its codes are compared where they are unique and
checked to be valid elsewhere; H, the combined output and the (straight-
through) backward meet the bf16 float tolerance."""
import numpy as np
import pytest
import torch

from mixture_experts_layer_59_b200 import binding as B
from mixture_experts_layer_59_b200 import synth
from oracle import moe_oracle as O

from helpers import BF16_TOL, assert_close, compare_plan, f64, fp32_router_logits, i64

pytestmark = pytest.mark.gpu


def sf_offset(r, kb, kchunks):
    """Byte offset of the scale of row r, 32-element K-block kb (the layout
    documented with the MXFP8 entry points)."""
    r, kb = np.asarray(r), np.asarray(kb)
    return ((r >> 7) * kchunks + (kb >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (kb & 3)


def u8(t):
    return t.detach().to("cpu").numpy().astype(np.uint8)


def expected_rows(q, se):
    """E4M3 codes of quantised rows (blocks along the last axis) and E8M0 codes."""
    return O.e4m3_encode(q), (se + 127).astype(np.uint8)


def test_mxfp8_weight_quantisation_bitexact():
    E, d, f = 3, 256, 384
    g = torch.Generator().manual_seed(40)
    w1 = (torch.randn(E, d, f, generator=g) * 0.02)
    w3 = (torch.randn(E, d, f, generator=g) * 0.02)
    w2 = (torch.randn(E, f, d, generator=g) * 0.02)
    w1[0, :32, 5] = 0.0                       # an all-zero block
    w1[1, 32:64, 7] *= 1e4                    # a block with a large maximum
    w3[2, :32, 9] = torch.tensor([1e-30] * 32)  # tiny values: scale at the E8M0 floor
    w2[0, 64:96, 3] = 448.0 * 2.0 ** 10       # elements that scale to exactly 448
    w1, w3, w2 = (w.to(torch.bfloat16) for w in (w1, w3, w2))
    wq = B.moe_mxfp8_quantize_weights(w1.cuda(), w3.cuda(), w2.cuda())
    torch.cuda.synchronize()
    w13q = u8(wq["w13q"]).reshape(E, 2 * f, d)
    w13s, w2s = u8(wq["w13s"]), u8(wq["w2s"])
    w2q = u8(wq["w2q"]).reshape(E, d, f)
    for e in range(E):
        for src, half in ((w1, 0), (w3, 1)):
            q, se = O.mx_quantize(f64(src[e]), 0)          # blocks along d, per column
            codes, scodes = expected_rows(q.T, se.T)        # [f, d], [f, d/32]
            for b in range(f // 128):
                rows = e * 2 * f + 256 * b + 128 * half + np.arange(128)
                cols = 128 * b + np.arange(128)
                np.testing.assert_array_equal(w13q[e, rows - e * 2 * f], codes[cols])
                kb = np.arange(d // 32)
                off = sf_offset(rows[:, None], kb[None, :], d // 128)
                np.testing.assert_array_equal(w13s[off], scodes[cols])
        q, se = O.mx_quantize(f64(w2[e]), 0)                # blocks along f, per column of d
        codes, scodes = expected_rows(q.T, se.T)            # [d, f], [d, f/32]
        np.testing.assert_array_equal(w2q[e], codes)
        rows = e * d + np.arange(d)
        off = sf_offset(rows[:, None], np.arange(f // 32)[None, :], f // 128)
        np.testing.assert_array_equal(w2s[off], scodes)
        # W1r / W3r: the weights' own [d, f] layout, blocks along f
        for src, qn, sn in ((w1, "w1rq", "w1rs"), (w3, "w3rq", "w3rs")):
            q, se = O.mx_quantize(f64(src[e]), 1)
            codes, scodes = expected_rows(q, se)            # [d, f], [d, f/32]
            np.testing.assert_array_equal(u8(wq[qn]).reshape(E, d, f)[e], codes)
            rows = e * d + np.arange(d)
            off = sf_offset(rows[:, None], np.arange(f // 32)[None, :], f // 128)
            np.testing.assert_array_equal(u8(wq[sn])[off], scodes)
    assert w13s[sf_offset(0 * 2 * f + 5, 0, d // 128)] == 0           # zero block -> code 0
    assert u8(wq["w2q"]).reshape(E, d, f)[0, 3, 64:96].tolist() == [0x7E] * 32   # 448


def _mx_layer(cfg, seed, round_mode):
    inp = synth.make_inputs(cfg, seed=seed, device="cuda")
    x, wg, w1, w3, w2, dout = (inp[n] for n in ("x", "w_gate", "w1", "w3", "w2", "dout"))
    bias = torch.linspace(0.5, -0.5, cfg.E)
    lg = fp32_router_logits(x, wg, bias)
    logits, idx, gate = B.moe_route(x, wg, cfg.k, logits_override=torch.from_numpy(lg).cuda())
    plan = B.moe_permute(idx, gate, logits, cfg.E, round_mode)
    wq = B.moe_mxfp8_quantize_weights(w1, w3, w2)
    ws = torch.empty(B.moe_ffn_fwd_mxfp8_workspace_size(cfg.T, cfg.d, cfg.f, cfg.E, cfg.k),
                     device="cuda", dtype=torch.uint8)
    H, Y = B.moe_expert_ffn_fwd_mxfp8(x, wq, plan, cfg.k, cfg.E, cfg.f, ws=ws)
    out = B.moe_combine(Y, plan["row_gate"], plan["slot_row"], plan["extra_row"], cfg.T, cfg.E,
                        cfg.k)
    g = B.moe_layer_bwd_mxfp8(dout, x, wg, w1, w3, w2, wq, idx, gate, plan, H)
    B.moe_check_status()
    torch.cuda.synchronize()
    fwd = O.layer_fwd(f64(x), f64(wg), f64(w1), f64(w3), f64(w2), cfg.k, round_mode=round_mode,
                      logits_override=lg.astype(np.float64), precision="mxfp8")
    bwd = O.layer_bwd(f64(dout), f64(x), f64(wg), f64(w1), f64(w3), f64(w2), fwd)
    return inp, plan, ws, H, out, g, fwd, bwd


def _ws_pieces(ws, cfg):
    cap = B.moe_row_capacity(cfg.T, cfg.E, cfg.k)
    capr = (cap + 127) // 128 * 128
    up = lambda n: (n + 255) // 256 * 256
    sizes = [capr * cfg.d, capr * cfg.d // 32, capr * cfg.f, capr * cfg.f // 32]
    raw, out, off = u8(ws), [], 0
    for n in sizes:
        out.append(raw[off:off + n])
        off += up(n)
    return out


@pytest.mark.parametrize("round_mode", [0, 1])
def test_mxfp8_forward_and_backward(round_mode):
    cfg = synth.MoEConfig("test", 1000, 256, 256, 8, 2, std=0.05)
    inp, plan, ws, H, out, g, fwd, bwd = _mx_layer(cfg, 41 + round_mode, round_mode)
    oplan = fwd["plan"]
    compare_plan(plan, oplan)
    R = oplan["R"]
    toks = oplan["row_token"][:R]
    live = toks >= 0
    xq, xs, aq, as_ = _ws_pieces(ws, cfg)
    d, f = cfg.d, cfg.f
    # quantised token rows: bit-exact codes and scales; padding rows zero
    q, se = O.mx_quantize(f64(inp["x"]), 1)
    codes, scodes = expected_rows(q, se)
    rows = np.arange(R)
    np.testing.assert_array_equal(xq.reshape(-1, d)[:R][live], codes[toks[live]])
    assert not xq.reshape(-1, d)[:R][~live].any()
    soff = sf_offset(rows[:, None], np.arange(d // 32)[None, :], d // 128)
    np.testing.assert_array_equal(xs[soff][live], scodes[toks[live]])
    assert not xs[soff][~live].any()
    # H from the block-scaled up-projection
    assert_close(f64(H)[:R][live], fwd["H"][:R][live], "H", BF16_TOL)
    # A's codes: from each side's own SwiGLU output -- identical almost
    # everywhere, elsewhere a neighbouring code of the same sign and scale
    qa, sea = O.mx_quantize(fwd["A"][:R], 1)
    acodes, ascodes = expected_rows(qa, sea)
    got = aq.reshape(-1, f)[:R]
    aoff = sf_offset(rows[:, None], np.arange(f // 32)[None, :], f // 128)
    gs = as_[aoff]
    same_scale = gs[live] == ascodes[live]
    assert same_scale.mean() > 0.999
    same = got[live] == acodes[live]
    assert same.mean() > 0.999, same.mean()
    mag = lambda c: (c.astype(np.int64) & 0x7F)
    ok_blocks = np.repeat(same_scale, 32, axis=1)
    diff = ~same & ok_blocks
    assert np.all(np.abs(mag(got[live][diff]) - mag(acodes[live][diff])) <= 1)
    # combined output and the backward (dX GEMM on MXFP8 operands)
    assert_close(out, fwd["out"], "out", BF16_TOL)
    assert_close(f64(g["dS"])[:R][live], bwd["dS"][:R][live], "dS", BF16_TOL)
    for n in ("dlogits", "dx", "dw_gate", "dw1", "dw3", "dw2"):
        assert_close(g[n], bwd[n], n, BF16_TOL)


def test_mxfp8_forward_differs_from_bf16_by_the_quantisation():
    """The MXFP8 output is not the bf16 output: their gap is of the size the
    format implies (a few E4M3 half-ulps), far above the parity tolerance."""
    cfg = synth.MoEConfig("test", 512, 256, 256, 8, 2, std=0.05)
    inp, plan, ws, H, out, g, fwd, bwd = _mx_layer(cfg, 43, 0)
    ref_bf16 = O.layer_fwd(f64(inp["x"]), f64(inp["w_gate"]), f64(inp["w1"]), f64(inp["w3"]),
                           f64(inp["w2"]), cfg.k, logits_override=fwd["logits"])["out"]
    rel = np.abs(f64(out) - ref_bf16).sum() / np.abs(ref_bf16).sum()
    assert 5e-3 < rel < 0.1, rel


@pytest.mark.parametrize("name,n_tok", [("coarse", 48), ("fine", 48)])
def test_mxfp8_full_size_sampled_tokens(name, n_tok):
    """Full workload sizes in the bench's launch configuration: out, dx,
    dlogits and dS of sampled tokens against the oracle's MXFP8 layer (each
    depends only on the token and its experts' weights)."""
    from test_gpu_full_configs import DeviceExperts
    cfg = synth.CONFIGS[name]
    T, E, k = cfg.T, cfg.E, cfg.k
    inp = synth.make_inputs(cfg, seed=0, device="cuda")
    x, wg, w1, w3, w2, dout = (inp[n] for n in ("x", "w_gate", "w1", "w3", "w2", "dout"))
    x64, wg64 = f64(x), f64(wg)
    lg = fp32_router_logits(x64, wg64, inp["logit_bias"])
    logits, idx, gate = B.moe_route(x, wg, k, logits_override=torch.from_numpy(lg).cuda())
    plan = B.moe_permute(idx, gate, logits, E)
    wq = B.moe_mxfp8_quantize_weights(w1, w3, w2)
    H, Y = B.moe_expert_ffn_fwd_mxfp8(x, wq, plan, k, E, cfg.f)
    out = B.moe_combine(Y, plan["row_gate"], plan["slot_row"], plan["extra_row"], T, E, k)
    g = B.moe_layer_bwd_mxfp8(dout, x, wg, w1, w3, w2, wq, idx, gate, plan, H)
    B.moe_check_status()
    torch.cuda.synchronize()
    lg64 = lg.astype(np.float64)
    _, oidx, ogate = O.route(None, None, k, logits_override=lg64)
    oplan = O.exact_plan(oidx, ogate, E)
    compare_plan(plan, oplan)
    fwd = dict(logits=lg64, idx=oidx, gate=ogate, plan=oplan, precision="mxfp8")
    rng = np.random.default_rng(7)
    tokens = sorted(set([0, T - 1] + list(rng.choice(T, n_tok - 2, replace=False))))
    s = O.sampled_tokens(tokens, f64(dout), x64, wg64, DeviceExperts(w1), DeviceExperts(w3),
                         DeviceExperts(w2), fwd)
    assert_close(f64(out)[tokens], np.stack([s["out"][t] for t in tokens]), "out", BF16_TOL)
    assert_close(f64(g["dx"])[tokens], np.stack([s["dx"][t] for t in tokens]), "dx", BF16_TOL)
    assert_close(f64(g["dlogits"])[tokens], np.stack([s["dlogits"][t] for t in tokens]),
                 "dlogits", BF16_TOL)
    rows = sorted(s["dS"])
    assert_close(f64(g["dS"])[rows], np.array([s["dS"][r] for r in rows]), "dS", BF16_TOL)


# ---------------------------------------------------------------- weight gradients on MXFP8
def _row_space(plan, width, g, gather_src=None):
    """A row-space bf16 matrix [cap, width] with zero padding rows, or None
    when gather_src (token rows) is given; the oracle's fp64 image [R, width]."""
    R = int(plan["offsets"][-1])
    tok = i64(plan["row_token"])[:R]
    if gather_src is not None:
        m = np.zeros((R, width))
        m[tok >= 0] = f64(gather_src)[tok[tok >= 0]]
        return None, m
    cap = plan["row_token"].numel()
    src = (torch.randn(cap, width, generator=g) * torch.exp(torch.randn(cap, 1, generator=g))
           ).to(torch.bfloat16)
    src[torch.from_numpy(np.concatenate([tok < 0, np.ones(cap - R, bool)]))] = 0
    return src.cuda(), f64(src)[:R]


@pytest.mark.parametrize("round_mode,gather", [(0, False), (1, False), (0, True), (1, True)])
def test_mxfp8_token_quantisation_bitexact(round_mode, gather):
    """moe_mxfp8_quantize_tokens: codes and scales of a row-space matrix
    quantised along its rows (blocks of 32 rows), bit for bit against the
    oracle's quantiser along axis 0; with gather_row, the rows come from
    token rows (padding rows zero)."""
    T, n, E, k = 700, 384, 8, 2
    g = torch.Generator().manual_seed(50 + round_mode + 2 * gather)
    lo = torch.randn(T, E, generator=g).cuda()
    logits, idx, gate = B.moe_route(None, None, k, logits_override=lo, T=T, E=E)
    plan = B.moe_permute(idx, gate, logits, E, round_mode)
    R = int(plan["offsets"][-1])
    capr = (B.moe_row_capacity(T, E, k) + 127) // 128 * 128
    if gather:
        x = (torch.randn(T, n, generator=g) * 3).to(torch.bfloat16).cuda()
        _, m = _row_space(plan, n, g, gather_src=x)
        q, sf = B.moe_mxfp8_quantize_tokens(x, plan["offsets"], capr, gather_row=plan["row_token"])
    else:
        src, m = _row_space(plan, n, g)
        q, sf = B.moe_mxfp8_quantize_tokens(src, plan["offsets"], capr)
    torch.cuda.synchronize()
    B.moe_check_status()
    oq, se = O.mx_quantize(m, 0)                         # [R, n], [R/32, n]
    codes, scodes = expected_rows(oq, se)
    np.testing.assert_array_equal(u8(q)[:, :R], codes.T)
    assert not u8(q)[:, R:].any()                        # rows past the plan untouched (zeros)
    kb = np.arange(R // 32)
    off = sf_offset(np.arange(n)[:, None], kb[None, :], capr // 128)
    np.testing.assert_array_equal(u8(sf)[off], scodes.T)


@pytest.mark.parametrize("round_mode", [0, 1])
def test_mxfp8_weight_gradients(round_mode):
    """Weight-gradient GEMMs on MXFP8 operands (wgrad=True) against the
    oracle's definition (operands quantised along tokens within each expert's
    segment); an expert without rows gets zero gradients; everything else in
    the backward is bit-identical to the bf16-wgrad run; and the MXFP8
    gradients differ from the bf16 ones by the size the format implies."""
    cfg = synth.MoEConfig("test", 900, 256, 256, 8, 2, std=0.05)
    inp = synth.make_inputs(cfg, seed=60 + round_mode, device="cuda")
    x, wg, w1, w3, w2, dout = (inp[n] for n in ("x", "w_gate", "w1", "w3", "w2", "dout"))
    bias = torch.linspace(0.5, -0.5, cfg.E)
    bias[5] = -1e4                                        # expert 5 receives no token
    lg = fp32_router_logits(x, wg, bias)
    logits, idx, gate = B.moe_route(x, wg, cfg.k, logits_override=torch.from_numpy(lg).cuda())
    plan = B.moe_permute(idx, gate, logits, cfg.E, round_mode)
    wq = B.moe_mxfp8_quantize_weights(w1, w3, w2)
    H, Y = B.moe_expert_ffn_fwd_mxfp8(x, wq, plan, cfg.k, cfg.E, cfg.f)
    g0 = B.moe_layer_bwd_mxfp8(dout, x, wg, w1, w3, w2, wq, idx, gate, plan, H)
    g1 = B.moe_layer_bwd_mxfp8(dout, x, wg, w1, w3, w2, wq, idx, gate, plan, H, wgrad=True)
    torch.cuda.synchronize()
    B.moe_check_status()
    assert int(plan["counts"][5]) == 0
    R = int(plan["offsets"][-1])
    for n in ("dx", "dw_gate", "dlogits"):
        assert torch.equal(g0[n], g1[n]), n
    live = plan["row_token"][:R] >= 0                   # (dS is written for live rows)
    assert torch.equal(g0["dS"][:R][live], g1["dS"][:R][live])
    for n in ("dw1", "dw3", "dw2"):
        assert not bool(g1[n][5].any()), n
    fwd = O.layer_fwd(f64(x), f64(wg), f64(w1), f64(w3), f64(w2), cfg.k, round_mode=round_mode,
                      logits_override=lg.astype(np.float64), precision="mxfp8")
    args = (f64(dout), f64(x), f64(wg), f64(w1), f64(w3), f64(w2), fwd)
    ref_mx = O.layer_bwd(*args, mx_wgrad_on=True)
    ref_bf = O.layer_bwd(*args)
    for n in ("dw1", "dw3", "dw2"):
        assert_close(g1[n], ref_mx[n], n, BF16_TOL)
        gap = np.abs(f64(g1[n]) - ref_bf[n]).sum() / np.abs(ref_bf[n]).sum()
        err = np.abs(f64(g1[n]) - ref_mx[n]).sum() / np.abs(ref_mx[n]).sum()
        assert gap > 5 * err and gap > 2e-3, (n, gap, err)


def test_mxfp8_token_quantisation_flags_rows_outside_its_buffers():
    """The quantiser's own checks: a gather row past the source (read as a
    zero row) and a plan longer than the output (skipped) are reported as
    device data check 0x140 and write nothing outside the buffers."""
    T, n, E, k = 300, 256, 4, 2
    g = torch.Generator().manual_seed(70)
    lo = torch.randn(T, E, generator=g).cuda()
    logits, idx, gate = B.moe_route(None, None, k, logits_override=lo, T=T, E=E)
    plan = B.moe_permute(idx, gate, logits, E)
    R = int(plan["offsets"][-1])
    capr = (B.moe_row_capacity(T, E, k) + 127) // 128 * 128
    x = torch.randn(T, n, generator=g).to(torch.bfloat16).cuda()
    bad = plan["row_token"].clone()
    r_bad = int(torch.nonzero(bad[:R] >= 0)[3])
    bad[r_bad] = T + 5
    q, sf = B.moe_mxfp8_quantize_tokens(x, plan["offsets"], capr, gather_row=bad)
    with pytest.raises(B.MoEError) as ei:
        B.moe_check_status()
    assert ei.value.code == B.MOE_ERR_DEVICE_CHECK and "0x140" in str(ei.value)
    good = bad.clone()
    good[r_bad] = -1                                      # what the kernel read instead
    q2, sf2 = B.moe_mxfp8_quantize_tokens(x, plan["offsets"], capr, gather_row=good)
    B.moe_check_status()
    assert torch.equal(q, q2) and torch.equal(sf, sf2)
    # a plan longer than the output rows: skipped, flagged
    q3, sf3 = B.moe_mxfp8_quantize_tokens(x, plan["offsets"], 128, gather_row=plan["row_token"])
    with pytest.raises(B.MoEError) as ei:
        B.moe_check_status()
    assert "0x140" in str(ei.value)
    assert not bool(q3.any()) and not bool(sf3.any())
