"""Pins for the CPU oracle: each check compares the oracle with something other
than itself (a library routine, brute force, a dense masked evaluation, a
closed form, finite differences, or the pages' worked example), so that a
dropped term, a wrong sign or index, or a transposed operand fails here."""
import itertools
import math
import os

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def _rand_layer(rng, T, d, f, E, scale=0.5):
    x = rng.standard_normal((T, d))
    wg = rng.standard_normal((d, E)) * scale
    w1 = rng.standard_normal((E, d, f)) * scale
    w3 = rng.standard_normal((E, d, f)) * scale
    w2 = rng.standard_normal((E, f, d)) * scale
    dout = rng.standard_normal((T, d))
    return x, wg, w1, w3, w2, dout


# ---------------------------------------------------------------- bf16 rounding

def test_bf16_round_matches_torch_conversion():
    rng = np.random.default_rng(1)
    v = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(2000) * 1e-30).astype(np.float32),
        (rng.standard_normal(2000) * 1e30).astype(np.float32),
        # exact halfway cases between bf16 neighbours (ties to even)
        np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8)], np.float32),
    ])
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.bf16_round(v.astype(np.float64)), ref)


def test_silu_and_grad_closed_forms():
    z = np.linspace(-8, 8, 101)
    np.testing.assert_allclose(O.silu(z), z / (1 + np.exp(-z)), rtol=1e-14, atol=1e-15)
    h = 1e-6
    num = (O.silu(z + h) - O.silu(z - h)) / (2 * h)
    np.testing.assert_allclose(O.silu_grad(z), num, rtol=1e-8, atol=1e-9)


# ---------------------------------------------------------------- routing

def test_route_matches_brute_force_sort_with_ties():
    rng = np.random.default_rng(2)
    T, E, k = 64, 8, 3
    logits = rng.integers(0, 3, size=(T, E)).astype(np.float64)  # many exact ties
    _, idx, gate = O.route(None, None, k, logits_override=logits)
    for t in range(T):
        brute = sorted(range(E), key=lambda e: (-logits[t, e], e))[:k]
        assert list(idx[t]) == brute
        vals = [logits[t, e] for e in brute]
        z = sum(math.exp(v) for v in vals)
        assert np.allclose(gate[t], [math.exp(v) / z for v in vals], rtol=1e-14)
    assert np.allclose(gate.sum(1), 1.0, rtol=1e-14)


def test_route_matches_torch_topk_softmax_without_ties():
    rng = np.random.default_rng(3)
    x, wg = rng.standard_normal((40, 16)), rng.standard_normal((16, 6))
    logits, idx, gate = O.route(x, wg, 2)
    tl = torch.from_numpy(x) @ torch.from_numpy(wg)
    v, i = torch.topk(tl, 2, dim=-1)
    np.testing.assert_allclose(logits, tl.numpy(), rtol=1e-13)
    np.testing.assert_array_equal(idx, i.numpy())
    np.testing.assert_allclose(gate, torch.softmax(v, -1).numpy(), rtol=1e-13)


def test_route_bias_shifts_logits():
    rng = np.random.default_rng(4)
    x, wg = rng.standard_normal((10, 8)), rng.standard_normal((8, 4))
    b = np.array([0.0, -1.0, 2.0, 0.5])
    logits, _, _ = O.route(x, wg, 2, logit_bias=b)
    np.testing.assert_allclose(logits, x @ wg + b, rtol=1e-13)


# ---------------------------------------------------------------- permutation

def test_exact_plan_matches_brute_force_dispatch():
    rng = np.random.default_rng(5)
    T, E, k, tile = 37, 5, 2, 4
    logits = rng.standard_normal((T, E))
    _, idx, gate = O.route(None, None, k, logits_override=logits)
    plan = O.exact_plan(idx, gate, E, tile)
    # brute force: per-expert lists in token order (the structure of a
    # dispatch into per-expert input lists), then tile-aligned placement
    lists = {e: [] for e in range(E)}
    for t in range(T):
        for j in range(k):
            lists[int(idx[t, j])].append((t, j))
    off = 0
    for e in range(E):
        assert plan["offsets"][e] == off
        assert plan["counts"][e] == len(lists[e])
        for i, (t, j) in enumerate(lists[e]):
            r = off + i
            assert plan["row_token"][r] == t
            assert plan["row_slot"][r] == t * k + j
            assert plan["slot_row"][t * k + j] == r
            assert plan["row_gate"][r] == gate[t, j]
        for r in range(off + len(lists[e]), off + -(-len(lists[e]) // tile) * tile):
            assert plan["row_token"][r] == -1 and plan["row_gate"][r] == 0
        off += -(-len(lists[e]) // tile) * tile
    assert plan["R"] == off


def test_exact_plan_invariants():
    rng = np.random.default_rng(6)
    T, E, k = 1000, 16, 4
    _, idx, gate = O.route(None, None, k, logits_override=rng.standard_normal((T, E)))
    plan = O.exact_plan(idx, gate, E)
    assert plan["counts"].sum() == T * k
    assert np.all(plan["offsets"] % O.TILE == 0)
    # slot_row is a bijection between the T*k slots and the live rows
    live = np.nonzero(plan["row_token"] >= 0)[0]
    assert len(live) == T * k
    assert sorted(plan["slot_row"]) == sorted(live)
    np.testing.assert_array_equal(plan["row_slot"][plan["slot_row"]], np.arange(T * k))
    for e in range(E):
        seg = plan["row_token"][plan["offsets"][e]:plan["offsets"][e] + plan["counts"][e]]
        assert np.all(np.diff(seg) > 0)


# ---------------------------------------------------------------- token rounding

def test_token_rounding_page_example():
    for cnt, tile, want in _golden("token_rounding_example.txt"):
        assert O.rounded_target([int(cnt)], T=10 ** 6, tile=int(tile))[0] == int(want)


def test_token_rounding_targets():
    c = np.array([0, 1, 63, 64, 65, 127, 128, 191, 192, 193, 300])
    r = O.rounded_target(c, T=10 ** 6, tile=128)
    np.testing.assert_array_equal(r, [0, 0, 0, 128, 128, 128, 128, 128, 256, 256, 256])
    assert np.all(np.abs(r - c) <= 64)
    # capped at the largest tile multiple not above T
    assert O.rounded_target([250], T=250, tile=128)[0] == 128


def test_rounded_plan_brute_force_subsets():
    """On tiny inputs the kept set of each shrunk expert is the size-r_e
    subset of its tokens with the largest total score, and the added set of
    each grown expert the size-(r_e - c_e) subset of the others with the
    largest total score; checked by enumerating every subset."""
    rng = np.random.default_rng(7)
    T, E, k, tile = 11, 3, 2, 4
    for trial in range(20):
        logits = rng.standard_normal((T, E))
        _, idx, gate = O.route(None, None, k, logits_override=logits)
        plan = O.rounded_plan(idx, logits, E, tile)
        counts = np.bincount(idx.ravel(), minlength=E)
        top = np.take_along_axis(logits, idx, 1)
        score = np.exp(logits) / np.exp(top).sum(1, keepdims=True)
        for e in range(E):
            assigned = [t for t in range(T) if e in idx[t]]
            others = [t for t in range(T) if e not in idx[t]]
            r = plan["target"][e]
            assert r % tile == 0 and abs(r - counts[e]) <= tile // 2
            members = set(int(t) for t in plan["row_token"][plan["offsets"][e]:plan["offsets"][e + 1]])
            assert len(members) == r
            if r <= counts[e]:
                best = max(itertools.combinations(assigned, r), key=lambda s: sum(score[t, e] for t in s))
                assert members == set(best)
            else:
                best = max(itertools.combinations(others, r - counts[e]),
                           key=lambda s: sum(score[t, e] for t in s))
                assert members == set(assigned) | set(best)
            seg = plan["row_gate"][plan["offsets"][e]:plan["offsets"][e + 1]]
            toks = plan["row_token"][plan["offsets"][e]:plan["offsets"][e + 1]]
            np.testing.assert_allclose(seg, score[toks, e], rtol=1e-13)
            assert np.all(np.diff(toks) > 0)


def test_rounded_plan_tie_rules():
    # every token has the same logits, so all keys of one expert are equal;
    # drops take the largest token ids, additions the smallest
    T, E, k, tile = 10, 3, 1, 4
    logits = np.tile(np.array([[1.0, 0.5, 0.0]]), (T, 1))
    logits[:6, 1] = 2.0          # tokens 0..5 choose expert 1, 6..9 choose 0
    _, idx, gate = O.route(None, None, k, logits_override=logits)
    plan = O.rounded_plan(idx, logits, E, tile)
    seg = lambda e: list(plan["row_token"][plan["offsets"][e]:plan["offsets"][e + 1]])
    assert seg(1) == [0, 1, 2, 3, 4, 5, 6, 7]   # 6 -> 8: adds the smallest ids
    assert seg(0) == [6, 7, 8, 9]               # 4 stays 4
    assert seg(2) == []                         # 0 stays 0
    logits2 = logits.copy()
    logits2[:, 2] = -1.0
    logits2[:7, 1] = 2.0                        # 7 tokens on expert 1 -> round to 8
    logits2[7:, 0] = 3.0                        # 3 on expert 0 -> round to 4
    _, idx2, _ = O.route(None, None, k, logits_override=logits2)
    p2 = O.rounded_plan(idx2, logits2, E, tile)
    s0 = list(p2["row_token"][p2["offsets"][0]:p2["offsets"][1]])
    assert s0 == [0, 7, 8, 9]


# ---------------------------------------------------------------- forward

def _dense_forward(x, wg, w1, w3, w2, k):
    """Every expert on every token, masked to the top-k (no permutation)."""
    logits = x @ wg
    T, E = logits.shape
    out = np.zeros_like(x)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-logits[t, e], e))[:k]
        z = sum(math.exp(logits[t, e] - logits[t, order[0]]) for e in order)
        for e in range(E):
            mask = e in order
            h1 = x[t] @ w1[e]
            h3 = x[t] @ w3[e]
            y = ((h1 / (1 + np.exp(-h1))) * h3) @ w2[e]
            g = math.exp(logits[t, e] - logits[t, order[0]]) / z if mask else 0.0
            out[t] += g * y
    return out


def test_forward_matches_dense_masked_evaluation():
    rng = np.random.default_rng(8)
    x, wg, w1, w3, w2, _ = _rand_layer(rng, 23, 6, 5, 4)
    fwd = O.layer_fwd(x, wg, w1, w3, w2, k=2, tile=4, staged=False)
    np.testing.assert_allclose(fwd["out"], _dense_forward(x, wg, w1, w3, w2, 2), rtol=1e-12, atol=1e-12)


def test_forward_matches_per_expert_masked_loop():
    """The structure of the Beam article's MoELayer: loop over the k slots and
    the experts with a boolean mask (here with SwiGLU experts)."""
    rng = np.random.default_rng(9)
    x, wg, w1, w3, w2, _ = _rand_layer(rng, 19, 4, 3, 5)
    k = 3
    scores = torch.from_numpy(x @ wg)
    vals, ids = scores.topk(k, dim=-1)
    vals = torch.softmax(vals, -1).numpy()
    ids = ids.numpy()
    out = np.zeros_like(x)
    for j in range(k):
        for e in range(5):
            m = ids[:, j] == e
            if m.any():
                h1 = x[m] @ w1[e]
                y = (h1 / (1 + np.exp(-h1)) * (x[m] @ w3[e])) @ w2[e]
                out[m] += vals[m, j][:, None] * y
    fwd = O.layer_fwd(x, wg, w1, w3, w2, k=k, tile=4, staged=False)
    np.testing.assert_allclose(fwd["out"], out, rtol=1e-12, atol=1e-12)


SILU1 = 0.7310585786300049      # silu(1) = 1 / (1 + e^-1)
DSILU1 = 0.9276705118714869     # silu'(1) = sigmoid(1) * (1 + (1 - sigmoid(1)))


def test_bf16_staging_points_on_hand_derived_scalars():
    """Each bf16 staging point of one expert's rows -- H, A and Y forward; A
    (recomputed), dH, s*A and dX_perm backward -- on 1 x 1 operands whose
    staged values were worked out by hand: bf16 keeps 8 significant bits, so
    values in [2^(e-1), 2^e) lie on a grid of 2^(e-8), ties to even.  Each
    case is chosen so that dropping or moving one rounding changes a result
    (the alternative is given beside each value)."""
    one = np.ones((1, 1))
    # H: h1 = 1 + 2^-9 is below 1 + 2^-8 (half the grid step at 1), so it is
    # stored as 1 and A = bf16(silu(1)) = bf16(187.15 / 256) = 187/256; from
    # the unrounded h1, silu(1 + 2^-9) = 187.62 / 256 would give 188/256.
    h1, h3, a, y = O.expert_rows_forward(one, one * (1 + 2.0 ** -9), one, one, staged=True)
    assert (h1[0, 0], h3[0, 0], a[0, 0], y[0, 0]) == (1.0, 1.0, 187 / 256, 187 / 256)
    # A and Y: with W2 = 9/16, A W2 = 187/256 * 9/16 = 210.375 * 2^-9, stored as
    # Y = 210/512; from an unrounded A, silu(1) * 9/16 = 210.55 * 2^-9 -> 211/512.
    _, _, a, y = O.expert_rows_forward(one, one, one, one * 9 / 16, staged=True)
    assert (a[0, 0], y[0, 0]) == (187 / 256, 210 / 512)
    _, _, a, y = O.expert_rows_forward(one, one, one, one * 9 / 16, staged=False)
    assert abs(a[0, 0] - SILU1) < 1e-15 and abs(y[0, 0] - SILU1 * 9 / 16) < 1e-15
    # Backward with x = 1, W1 = 1, W3 = 5/4, W2 = 1/4, dO = 5/4, gate g = 3/8:
    # h1 = 1, h3 = 5/4, A = bf16(silu(1) * 5/4 = 233.94 / 256) = 234/256.
    w3, w2, dout, g = one * 5 / 4, one / 4, one * 5 / 4, np.array([3 / 8])
    ds, da1, da3, ga, dxp = O.expert_rows_backward(dout, g, one, w3, one, w3, w2, staged=True)
    # dS = <dA', A> with dA' = dO W2^T = 5/16: 5/16 * 234/256 = 585/2048
    # (0.285567 from an unrounded A)
    assert ds[0] == 585 / 2048
    # dA = g dA' = 15/128; dH3 = bf16(dA silu(1) = 175.45 * 2^-11) = 175/2048
    assert da3[0, 0] == 175 / 2048
    # dH1 = bf16(dA h3 silu'(1) = 139.15 * 2^-10) = 139/1024
    assert da1[0, 0] == 139 / 1024
    # s*A = bf16(3/8 * 234/256 = 175.5 * 2^-9): a tie, to even -> 176/512
    # (175/512 from an unrounded A, 175.45 * 2^-9)
    assert ga[0, 0] == 176 / 512
    # dX_perm = bf16(dH1 W1 + dH3 W3 = 139/1024 + 175/2048 * 5/4 = 248.375 * 2^-10)
    # = 248/1024 (from unrounded dH1, dH3: 248.81 * 2^-10 -> 249/1024)
    assert dxp[0, 0] == 248 / 1024
    ds, da1, da3, ga, dxp = O.expert_rows_backward(dout, g, one, w3, one, w3, w2, staged=False)
    assert abs(ds[0] - 5 / 16 * SILU1 * 5 / 4) < 1e-15
    assert abs(da1[0, 0] - 15 / 128 * 5 / 4 * DSILU1) < 1e-15
    assert abs(dxp[0, 0] - (15 / 128 * 5 / 4 * DSILU1 + 15 / 128 * SILU1 * 5 / 4)) < 1e-15


def test_staged_forward_close_to_ideal():
    rng = np.random.default_rng(10)
    x, wg, w1, w3, w2, _ = _rand_layer(rng, 50, 32, 16, 4, scale=0.2)
    a = O.layer_fwd(x, wg, w1, w3, w2, k=2, staged=False)["out"]
    b = O.layer_fwd(x, wg, w1, w3, w2, k=2, staged=True)["out"]
    err = np.abs(a - b).sum() / np.abs(a).sum()
    assert 1e-5 < err < 2e-2


# ---------------------------------------------------------------- backward

def test_two_expert_hand_example():
    want = {n: float(v) for n, v in _golden("two_expert_example.txt")}
    x = np.array([[1.0]])
    wg = np.array([[math.log(3.0), 0.0]])
    w1 = np.array([[[0.0]], [[1.0]]])
    w3 = np.array([[[1.0]], [[2.0]]])
    w2 = np.array([[[1.0]], [[1.0]]])
    dout = np.array([[1.0]])
    fwd = O.layer_fwd(x, wg, w1, w3, w2, k=2, tile=1, staged=False)
    bwd = O.layer_bwd(dout, x, wg, w1, w3, w2, fwd, staged=False)
    assert abs(fwd["out"][0, 0] - want["out"]) < 1e-9
    rows = fwd["plan"]["slot_row"]      # slot 0 -> expert 0, slot 1 -> expert 1
    assert abs(bwd["dS"][rows[0]] - want["dS0"]) < 1e-9
    assert abs(bwd["dS"][rows[1]] - want["dS1"]) < 1e-9
    for n, arr in (("dw_gate", bwd["dw_gate"][0]), ("dw1_", bwd["dw1"][:, 0, 0]),
                   ("dw3_", bwd["dw3"][:, 0, 0]), ("dw2_", bwd["dw2"][:, 0, 0])):
        for e in range(2):
            assert abs(arr[e] - want[f"{n}{e}"]) < 1e-9, (n, e)
    assert abs(bwd["dx"][0, 0] - want["dx"]) < 1e-9


def _loss(params, dout, k, tile, round_mode, gate_mode=0, capacity=None, noise=None):
    x, wg, w1, w3, w2 = params
    fwd = O.layer_fwd(x, wg, w1, w3, w2, k=k, tile=tile, round_mode=round_mode, staged=False,
                      gate_mode=gate_mode, capacity=capacity, logit_noise=noise)
    return float(np.sum(fwd["out"] * dout)), fwd


@pytest.mark.parametrize("round_mode,gate_mode,capacity,noisy", [
    (0, 0, None, 0), (1, 0, None, 0), (0, 1, None, 0), (1, 1, None, 0), (2, 0, 3, 0), (2, 1, 3, 0),
    (0, 0, None, 1), (1, 1, None, 1)])
def test_backward_matches_central_differences(round_mode, gate_mode, capacity, noisy):
    rng = np.random.default_rng(11 + round_mode + 10 * gate_mode + 100 * noisy)
    T, d, f, E, k, tile = 9, 4, 3, 4, 2, 4
    x, wg, w1, w3, w2, dout = _rand_layer(rng, T, d, f, E)
    params = [x, wg, w1, w3, w2]
    noise = rng.standard_normal((T, E)) if noisy else None
    _, fwd = _loss(params, dout, k, tile, round_mode, gate_mode, capacity, noise)
    if noisy:   # the noise changes the routing of some token
        assert not np.array_equal(fwd["idx"], _loss(params, dout, k, tile, round_mode,
                                                     gate_mode, capacity)[1]["idx"])
    if round_mode:
        assert fwd["plan"]["dropped"].any() or fwd["plan"]["added"].any()
    bwd = O.layer_bwd(dout, x, wg, w1, w3, w2, fwd, staged=False)
    grads = [bwd["dx"], bwd["dw_gate"], bwd["dw1"], bwd["dw3"], bwd["dw2"]]
    h = 1e-6
    for p, g in zip(params, grads):
        num = np.zeros_like(p)
        for i in np.ndindex(p.shape):
            old = p[i]
            p[i] = old + h
            lp, fp = _loss(params, dout, k, tile, round_mode, gate_mode, capacity, noise)
            p[i] = old - h
            lm, fm = _loss(params, dout, k, tile, round_mode, gate_mode, capacity, noise)
            p[i] = old
            # the discrete routing must not change under the probe
            assert np.array_equal(fp["idx"], fwd["idx"]) and np.array_equal(fm["idx"], fwd["idx"])
            assert np.array_equal(fp["plan"]["row_token"], fwd["plan"]["row_token"])
            num[i] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=1e-5, atol=1e-7)


def test_dS_identity_inner_products():
    """<dA', A> computed by the oracle equals <dO, Y> (the quantity it replaces)."""
    rng = np.random.default_rng(12)
    x, wg, w1, w3, w2, dout = _rand_layer(rng, 30, 8, 6, 4)
    fwd = O.layer_fwd(x, wg, w1, w3, w2, k=2, tile=4, staged=False)
    bwd = O.layer_bwd(dout, x, wg, w1, w3, w2, fwd, staged=False)
    rows = np.nonzero(fwd["plan"]["row_token"] >= 0)[0]
    toks = fwd["plan"]["row_token"][rows]
    np.testing.assert_allclose(bwd["dS"][rows], np.sum(dout[toks] * fwd["Y"][rows], 1), rtol=1e-11)


def test_router_grad_rows_sum_to_zero_in_exact_mode():
    """Softmax over the top-k is shift invariant, so each token's dlogits sums
    to zero over its k experts and vanishes elsewhere."""
    rng = np.random.default_rng(13)
    x, wg, w1, w3, w2, dout = _rand_layer(rng, 25, 6, 4, 5)
    fwd = O.layer_fwd(x, wg, w1, w3, w2, k=2, tile=4, staged=False)
    bwd = O.layer_bwd(dout, x, wg, w1, w3, w2, fwd, staged=False)
    np.testing.assert_allclose(bwd["dlogits"].sum(1), 0, atol=1e-12)
    mask = np.ones_like(bwd["dlogits"], bool)
    mask[np.arange(25)[:, None], fwd["idx"]] = False
    assert np.all(bwd["dlogits"][mask] == 0)


def test_sampled_views_equal_full_layer():
    rng = np.random.default_rng(14)
    x, wg, w1, w3, w2, dout = _rand_layer(rng, 40, 8, 6, 4, scale=0.3)
    for rm in (0, 1):
        fwd = O.layer_fwd(x, wg, w1, w3, w2, k=2, tile=4, round_mode=rm)
        bwd = O.layer_bwd(dout, x, wg, w1, w3, w2, fwd)
        s = O.sampled_tokens([0, 7, 39], dout, x, wg, w1, w3, w2, fwd)
        for t in (0, 7, 39):
            np.testing.assert_allclose(s["out"][t], fwd["out"][t], rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(s["dx"][t], bwd["dx"][t], rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(s["dlogits"][t], bwd["dlogits"][t], rtol=1e-12, atol=1e-14)
        ge = O.sampled_expert_grads([1, 3], dout, x, w1, w3, w2, fwd)
        for e in (1, 3):
            for n in ("dw1", "dw3", "dw2"):
                np.testing.assert_allclose(ge[e][n], bwd[n][e], rtol=1e-12, atol=1e-14)


def test_rounded_plan_drop_tie_takes_largest_token():
    # 5 tokens on expert 0 with equal keys, tile 4 -> 4 rows: token 4 is dropped
    T, E, k, tile = 8, 2, 1, 4
    logits = np.zeros((T, E))
    logits[:5, 0] = 1.0
    logits[5:, 1] = 1.0
    _, idx, gate = O.route(None, None, k, logits_override=logits)
    plan = O.rounded_plan(idx, logits, E, tile)
    assert list(plan["row_token"][0:4]) == [0, 1, 2, 3]
    assert plan["slot_row"][4] == -1 and plan["dropped"][4, 0]


def test_expert_grad_slices_equal_full_grads():
    rng = np.random.default_rng(15)
    x, wg, w1, w3, w2, dout = _rand_layer(rng, 60, 8, 12, 3, scale=0.3)
    for rm in (0, 1):
        fwd = O.layer_fwd(x, wg, w1, w3, w2, k=2, tile=4, round_mode=rm)
        bwd = O.layer_bwd(dout, x, wg, w1, w3, w2, fwd)
        cols = [0, 5, 11]
        for e in range(3):
            sl = O.expert_grad_slices(e, cols, dout, x, w1[e], w3[e], w2[e], fwd)
            np.testing.assert_allclose(sl["dw1"], bwd["dw1"][e][:, cols], rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(sl["dw3"], bwd["dw3"][e][:, cols], rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(sl["dw2"], bwd["dw2"][e][cols, :], rtol=1e-12, atol=1e-14)


def test_rows_compute_accepts_per_expert_weight_access():
    rng = np.random.default_rng(16)
    x, wg, w1, w3, w2, dout = _rand_layer(rng, 30, 8, 6, 4, scale=0.3)
    fwd = O.layer_fwd(x, wg, w1, w3, w2, k=2, tile=4)

    class Lazy:
        def __init__(self, a):
            self.a = a

        def __getitem__(self, e):
            return self.a[e].astype(np.float32)

    s1 = O.sampled_tokens([3, 9], dout, x, wg, w1, w3, w2, fwd)
    s2 = O.sampled_tokens([3, 9], dout, x, wg, Lazy(w1), Lazy(w3), Lazy(w2), fwd)
    for t in (3, 9):
        np.testing.assert_allclose(s1["dx"][t], s2["dx"][t], rtol=1e-6, atol=1e-9)


# ---------------------------------------------------------------- balance loss

def test_balance_loss_closed_form_uniform_and_collapsed():
    # perfectly balanced routing: every expert gets the same importance -> 0
    T, E, k = 8, 4, 1
    idx = np.array([[t % E] for t in range(T)])
    gate = np.ones((T, k))
    r = O.balance_loss(idx, gate, E, lam=0.5)
    assert r["loss"] == 0 and r["count_mse"] == 0 and r["max_share"] == 0.25
    # every token on expert 0: importance = [1,0,0,0], mean 1/4, var 3/16,
    # CV^2 = (3/16)/(1/16) = 3 = E - 1
    idx = np.zeros((T, 1), int)
    r = O.balance_loss(idx, gate, E, lam=2.0)
    assert abs(r["loss"] - 2.0 * 3) < 1e-12
    assert r["max_share"] == 1.0 and abs(r["count_cv2"] - 3) < 1e-12
    # counts [8,0,0,0]: mean 2, squared deviations 36,4,4,4 -> mse 12
    assert abs(r["count_mse"] - 12) < 1e-12


def test_balance_loss_matches_torch_autograd():
    rng = np.random.default_rng(17)
    T, E, k = 20, 6, 2
    logits = rng.standard_normal((T, E))
    _, idx, gate = O.route(None, None, k, logits_override=logits)
    r = O.balance_loss(idx, gate, E, lam=0.3)
    g = torch.tensor(gate, requires_grad=True)
    G = torch.zeros(T, E, dtype=torch.float64).scatter(1, torch.tensor(idx, dtype=torch.int64), g)
    imp = G.mean(0)
    loss = 0.3 * imp.var(unbiased=False) / imp.mean() ** 2
    loss.backward()
    assert abs(loss.item() - r["loss"]) < 1e-12
    np.testing.assert_allclose(r["dgate"], g.grad.numpy(), rtol=1e-10, atol=1e-14)
    np.testing.assert_allclose(r["importance"], imp.detach().numpy(), rtol=1e-12)


def test_gate_grad_to_logits_matches_finite_differences():
    rng = np.random.default_rng(18)
    T, E, k = 6, 5, 3
    logits = rng.standard_normal((T, E))
    _, idx, gate = O.route(None, None, k, logits_override=logits)
    a = rng.standard_normal((T, k))
    dl = O.gate_grad_to_logits(idx, gate, a, E)
    h = 1e-6
    for t in range(T):
        for e in range(E):
            lp, lm = logits.copy(), logits.copy()
            lp[t, e] += h
            lm[t, e] -= h
            gp = O.route(None, None, k, logits_override=lp)[2]
            gm = O.route(None, None, k, logits_override=lm)[2]
            num = ((gp - gm) * a).sum() / (2 * h)
            assert abs(num - dl[t, e]) < 1e-7


def test_layer_with_balance_loss_matches_central_differences():
    """Total loss = <dO, O> + lambda CV^2: gradients through both terms."""
    rng = np.random.default_rng(19)
    T, d, f, E, k, tile, lam = 9, 4, 3, 4, 2, 4, 0.7
    x, wg, w1, w3, w2, dout = _rand_layer(rng, T, d, f, E)

    def total(xx, wgg):
        fwd = O.layer_fwd(xx, wgg, w1, w3, w2, k=k, tile=tile, staged=False)
        return float(np.sum(fwd["out"] * dout)) + O.balance_loss(fwd["idx"], fwd["gate"], E, lam)["loss"], fwd

    _, fwd = total(x, wg)
    bl = O.balance_loss(fwd["idx"], fwd["gate"], E, lam)
    extra = O.gate_grad_to_logits(fwd["idx"], fwd["gate"], bl["dgate"], E)
    bwd = O.layer_bwd(dout, x, wg, w1, w3, w2, fwd, staged=False, extra_dlogits=extra)
    h = 1e-6
    for p, g in ((x, bwd["dx"]), (wg, bwd["dw_gate"])):
        num = np.zeros_like(p)
        for i in np.ndindex(p.shape):
            old = p[i]
            p[i] = old + h
            lp, fp = total(x, wg)
            p[i] = old - h
            lm, fm = total(x, wg)
            p[i] = old
            assert np.array_equal(fp["idx"], fwd["idx"]) and np.array_equal(fm["idx"], fwd["idx"])
            num[i] = (lp - lm) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=1e-5, atol=1e-7)



# ---------------------------------------------------------------- routing variants

def test_route_softmax_then_topk_matches_library():
    """Gate mode 1: softmax over all E logits, then the k largest without
    renormalisation (the gating of the Trinity commentary's challenge 1)."""
    rng = np.random.default_rng(20)
    x, wg = rng.standard_normal((30, 16)), rng.standard_normal((16, 4))
    _, idx, gate = O.route(x, wg, 2, gate_mode=1)
    p = torch.softmax(torch.from_numpy(x @ wg), -1)
    v, i = torch.topk(p, 2, dim=-1)
    np.testing.assert_array_equal(idx, i.numpy())
    np.testing.assert_allclose(gate, v.numpy(), rtol=1e-13)
    assert np.all(gate.sum(1) < 1.0)


def test_capacity_plan_brute_force_subsets():
    rng = np.random.default_rng(21)
    T, E, k, tile = 12, 3, 2, 4
    for trial in range(20):
        for gate_mode in (0, 1):
            logits = rng.standard_normal((T, E))
            _, idx, gate = O.route(None, None, k, logits_override=logits, gate_mode=gate_mode)
            C = 5
            plan = O.make_plan(idx, gate, logits, E, tile, round_mode=2, gate_mode=gate_mode,
                               capacity=C)
            counts = np.bincount(idx.ravel(), minlength=E)
            key = O.rounding_keys(logits, idx, gate_mode)
            assert not plan["added"].any()
            for e in range(E):
                lo, hi = plan["offsets"][e], plan["offsets"][e + 1]
                assert lo % tile == 0 and hi % tile == 0
                members = [int(t) for t in plan["row_token"][lo:hi] if t >= 0]
                assigned = [t for t in range(T) if e in idx[t]]
                keep = min(counts[e], C)
                assert len(members) == keep
                best = max(itertools.combinations(assigned, keep), key=lambda s: sum(key[t, e] for t in s))
                assert set(members) == set(best)
                for r in range(lo, hi):
                    t = plan["row_token"][r]
                    if t >= 0:
                        j = list(idx[t]).index(e)
                        assert abs(plan["row_gate"][r] - gate[t, j]) <= 1e-12 * gate[t, j]


def test_gate_grad_to_logits_mode1_matches_finite_differences():
    rng = np.random.default_rng(22)
    T, E, k = 5, 6, 2
    logits = rng.standard_normal((T, E))
    _, idx, gate = O.route(None, None, k, logits_override=logits, gate_mode=1)
    a = rng.standard_normal((T, k))
    dl = O.gate_grad_to_logits(idx, gate, a, E, gate_mode=1, logits=logits)
    h = 1e-6
    for t in range(T):
        for e in range(E):
            lp, lm = logits.copy(), logits.copy()
            lp[t, e] += h
            lm[t, e] -= h
            gp = O.route(None, None, k, logits_override=lp, gate_mode=1)[2]
            gm = O.route(None, None, k, logits_override=lm, gate_mode=1)[2]
            assert abs(((gp - gm) * a).sum() / (2 * h) - dl[t, e]) < 1e-7


def test_noisy_routing_special_cases():
    """Zero noise is no noise; a dominant noise on one expert makes every token
    choose it first, with gate -> 1 under the all-E softmax, and leaves the
    choice of the other k-1 experts to the clean logits."""
    rng = np.random.default_rng(23)
    T, d, E, k = 40, 8, 6, 3
    x, wg = rng.standard_normal((T, d)), rng.standard_normal((d, E))
    base = O.route(x, wg, k)
    zero = O.route(x, wg, k, logit_noise=np.zeros((T, E)))
    for a, b in zip(base, zero):
        np.testing.assert_array_equal(a, b)
    eps = np.zeros((T, E))
    eps[:, 4] = 80.0
    lg, idx, gate = O.route(x, wg, k, gate_mode=1, logit_noise=eps)
    assert np.all(idx[:, 0] == 4)
    np.testing.assert_allclose(gate[:, 0], 1.0, rtol=1e-12)
    clean = x @ wg
    for t in range(T):
        rest = [e for e in np.argsort(-clean[t], kind="stable") if e != 4][:k - 1]
        assert list(idx[t, 1:]) == rest
    np.testing.assert_allclose(lg, clean + eps, rtol=1e-15)


# ---------------------------------------------------------------- MXFP8 (OCP MX, E4M3 elements)

def _e4m3_torch(v):
    t = torch.from_numpy(np.asarray(v, np.float32))
    return t.to(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_e4m3_round_matches_torch_below_overflow():
    """Round-to-nearest-even on the E4M3 grid, against torch's float8_e4m3fn
    conversion, for normal, subnormal and exact-midpoint inputs (|v| < 464,
    where rounding never overflows)."""
    rng = np.random.default_rng(30)
    mant = rng.uniform(1.0, 2.0, 4000)
    ex = rng.integers(-12, 9, 4000)
    v = (mant * np.ldexp(1.0, ex)).astype(np.float32).astype(np.float64)
    v *= np.where(rng.random(4000) < 0.5, -1.0, 1.0)
    grid = np.unique(np.abs(O.e4m3_decode(np.arange(0, 0x7F))))
    mids = (grid[1:] + grid[:-1]) / 2                    # exact ties
    v = np.concatenate([v, mids, -mids])
    v = v[np.abs(v) < 464]
    np.testing.assert_array_equal(O.e4m3_round(v), _e4m3_torch(v))


def test_e4m3_code_table():
    """All 256 codes: decode agrees with torch's float8_e4m3fn bit pattern,
    encode inverts decode, and the extremes are the format's."""
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    dec = O.e4m3_decode(codes)
    np.testing.assert_array_equal(np.isnan(dec), np.isnan(ref))
    ok = ~np.isnan(dec)
    np.testing.assert_array_equal(dec[ok], ref[ok])
    np.testing.assert_array_equal(O.e4m3_encode(dec[ok]), codes[ok])
    assert O.e4m3_decode(0x7E) == 448 and O.e4m3_decode(0x08) == 2.0 ** -6
    assert O.e4m3_decode(0x01) == 2.0 ** -9 and O.e4m3_decode(0x80) == 0 and np.signbit(O.e4m3_decode(0x80))


def test_e4m3_saturates_to_448():
    v = np.array([448, 463.99, 464, 465, 479.9, 480, 512, 1e6, 3e38])
    np.testing.assert_array_equal(O.e4m3_round(v), np.minimum(_e4m3_torch(np.minimum(v, 448)), 448))
    np.testing.assert_array_equal(O.e4m3_round(v), np.full(v.shape, 448.0))
    np.testing.assert_array_equal(O.e4m3_round(-v), np.full(v.shape, -448.0))


def test_mx_shared_exponent_closed_form():
    """2^se is the largest power of two with amax / 2^se >= 256 (so the block
    maximum scales into [256, 512)); all-zero blocks and tiny maxima take the
    E8M0 floor -127, huge maxima its ceiling 127."""
    rng = np.random.default_rng(31)
    amax = np.exp(rng.uniform(-60, 60, 2000))
    se = O.mx_shared_exp(amax)
    r = amax / np.ldexp(1.0, se)
    assert np.all((r >= 256) & (r < 512))
    assert np.all(se == np.floor(np.log2(amax / 256.0)))
    np.testing.assert_array_equal(O.mx_shared_exp(np.array([0.0, 2.0 ** -140, 2.0 ** 140])),
                                  [-127, -127, 127])
    np.testing.assert_array_equal(O.mx_shared_exp(np.array([1.0, 256.0, 511.999, 512.0])),
                                  [-8, 0, 0, 1])


def test_mx_quantize_error_bound_and_idempotence():
    """Each element is the E4M3 rounding of v / 2^se: error <= 2^-4 |v| in the
    normal range, <= 2^(se-10) in the subnormal range, and only elements
    that scale to >= 464 saturate.  Blocks run along the requested axis."""
    rng = np.random.default_rng(32)
    a = rng.standard_normal((6, 96)) * np.exp(rng.uniform(-8, 8, (6, 1)))
    a[2, 32:64] = 0.0                                     # an all-zero block
    a[3, :5] *= 1e-6                                      # subnormal-range elements
    for axis, arr in ((1, a), (0, a.T.copy())):
        q, se = O.mx_quantize(arr, axis)
        assert se.shape == ((6, 3) if axis == 1 else (3, 6))
        deq = O.mx_dequantize(q, se, axis)
        scale = np.repeat(np.ldexp(1.0, se), 32, axis=axis)
        s = arr / scale
        err = np.abs(deq - arr) / scale
        sat = np.abs(s) >= 464
        assert np.all(err[~sat] <= np.maximum(np.abs(s[~sat]) * 2.0 ** -4, 2.0 ** -10) * (1 + 1e-12))
        assert np.all(np.abs(q[sat]) == 448)
        np.testing.assert_array_equal(O.mx_fake_quant(deq, axis), deq)   # idempotent
    q, se = O.mx_quantize(a, 1)
    assert se[2, 1] == -127 and np.all(q[2, 32:64] == 0)


def test_mxfp8_layer_equals_bf16_layer_on_the_mx_grid():
    """With x, W1, W3 already on the MXFP8 grid the quantised up-projection is
    exact, so H equals the unquantised layer's; Y then uses the MXFP8 image of
    A and W2; the backward reads the MXFP8 forward's H."""
    rng = np.random.default_rng(33)
    T, d, f, E, k = 24, 64, 64, 4, 2
    x, wg, w1, w3, w2, dout = _rand_layer(rng, T, d, f, E)
    x, w1, w3 = O.mx_fake_quant(x, 1), O.mx_fake_quant(w1, 1), O.mx_fake_quant(w3, 1)
    a = O.layer_fwd(x, wg, w1, w3, w2, k, tile=4, staged=False)
    b = O.layer_fwd(x, wg, w1, w3, w2, k, tile=4, staged=False, precision="mxfp8")
    np.testing.assert_array_equal(a["H"], b["H"])
    R = b["plan"]["R"]
    for r in range(R):
        e, t = O.row_expert(b["plan"], [r])[0], b["plan"]["row_token"][r]
        if t < 0:
            continue
        want = O.mx_fake_quant(a["A"][r:r + 1], 1) @ O.mx_fake_quant(w2[e], 0)
        np.testing.assert_allclose(b["Y"][r], want[0], rtol=1e-13, atol=1e-15)
    assert np.abs(b["Y"] - a["Y"]).max() > 0             # A and W2 are not on the grid
    ga = O.layer_bwd(dout, x, wg, w1, w3, w2, a, staged=False)
    gb = O.layer_bwd(dout, x, wg, w1, w3, w2, b, staged=False)
    for n in ("dw1", "dw3", "dw2", "dS", "dlogits"):   # same H, straight-through backward
        np.testing.assert_allclose(gb[n], ga[n], rtol=1e-12, atol=1e-12)
    # dX_perm takes MXFP8 dH and W1/W3 (blocks along f): exactly the dH rows
    # of the unquantised backward, quantised, times the quantised weights
    f = w1.shape[2]
    for r in range(R):
        e, t = O.row_expert(b["plan"], [r])[0], b["plan"]["row_token"][r]
        if t < 0:
            continue
        dh = ga["dH"][r:r + 1]
        want = (O.mx_fake_quant(dh[:, :f], 1) @ O.mx_fake_quant(w1[e], 1).T
                + O.mx_fake_quant(dh[:, f:], 1) @ O.mx_fake_quant(w3[e], 1).T)
        np.testing.assert_allclose(gb["dXp"][r], want[0], rtol=1e-12, atol=1e-14)



def test_mx_wgrad_blocks_run_along_tokens_within_the_segment():
    """MXFP8 weight gradient: operands quantised in blocks of 32 consecutive
    token rows.  Column 0 of a holds 2^10 in row 31 and 2^-10 in the other
    rows of that block: the block's scale is 2^(10-8), so 2^-10 / 2^2 = 2^-12
    falls below half the smallest E4M3 subnormal (2^-9) and rounds to zero.
    Rows 32..63 form their own block (scale 2^(-10-8)) and keep 2^-10 exactly.
    With b = ones the gradient is then 2^10 + 32 * 2^-10 in closed form,
    against 2^10 + 63 * 2^-10 unquantised.  Column 1 of a is 3 everywhere
    (exact in E4M3 at any shared scale): 64 * 3."""
    a = np.full((64, 2), 2.0 ** -10)
    a[31, 0] = 2.0 ** 10
    a[:, 1] = 3.0
    b = np.ones((64, 1))
    got = O.mx_wgrad(a, b)
    assert got.shape == (2, 1)
    assert got[0, 0] == 2.0 ** 10 + 32 * 2.0 ** -10
    assert got[1, 0] == 64 * 3.0
    assert (a.T @ b)[0, 0] == 2.0 ** 10 + 63 * 2.0 ** -10
    # the segment helper puts live rows where they sit, zeros in padding rows
    live = np.array([True, False, True, True])
    seg = O._segment(np.array([[1.0], [2.0], [3.0]]), live, 1)
    np.testing.assert_array_equal(seg[:, 0], [1.0, 0.0, 2.0, 3.0])


def test_layer_bwd_mx_wgrad_close_to_the_unquantised_gradient():
    """The MXFP8 weight gradients differ from the straight-through (bf16)
    ones by the format's rounding: relative error of a few E4M3 half-ulps
    (2^-4) in aggregate, never zero, and nothing else in the backward moves."""
    T, d, f, E, k = 96, 64, 32, 4, 2
    rng = np.random.default_rng(35)
    x = rng.standard_normal((T, d))
    wg = 0.3 * rng.standard_normal((d, E))
    w1, w3 = 0.2 * rng.standard_normal((E, d, f)), 0.2 * rng.standard_normal((E, d, f))
    w2 = 0.2 * rng.standard_normal((E, f, d))
    dout = rng.standard_normal((T, d))
    fwd = O.layer_fwd(x, wg, w1, w3, w2, k, tile=32, staged=False)
    ref = O.layer_bwd(dout, x, wg, w1, w3, w2, fwd, staged=False)
    mx = O.layer_bwd(dout, x, wg, w1, w3, w2, fwd, staged=False, mx_wgrad_on=True)
    for n in ("dw1", "dw3", "dw2"):
        rel = np.abs(mx[n] - ref[n]).sum() / np.abs(ref[n]).sum()
        assert 1e-4 < rel < 2 ** -4, (n, rel)
    for n in ("dx", "dw_gate", "dlogits", "dS"):
        np.testing.assert_array_equal(mx[n], ref[n])


def test_mx_fake_quant_matches_torch_float8_along_either_axis():
    """The MXFP8 image of a matrix, blocks along rows or columns, against an
    independent torch construction: per-block maximum, scale 2^(e-9) from
    torch.frexp (max = m 2^e, m in [0.5, 1)), clamp to +-448 and torch's
    float8_e4m3fn rounding."""
    rng = np.random.default_rng(34)
    a = rng.standard_normal((64, 96)) * np.exp(rng.uniform(-6, 6, (64, 1)))
    for axis in (0, 1):
        t = torch.from_numpy(np.moveaxis(a, axis, -1).copy())
        blk = t.reshape(*t.shape[:-1], -1, 32)
        amax = blk.abs().amax(-1, keepdim=True)
        _, ex = torch.frexp(amax)
        scale = torch.pow(2.0, (ex - 9).to(torch.float64))
        q = (blk / scale).clamp(-448, 448).to(torch.float8_e4m3fn).to(torch.float64)
        ref = np.moveaxis((q * scale).reshape(t.shape).numpy(), -1, axis)
        np.testing.assert_array_equal(O.mx_fake_quant(a, axis), ref)


def test_balanced_routing_gives_equal_expert_loads():
    """The `balanced` synthetic router sends exactly T*k/E rows to every
    expert (each token's k experts distinct), so grouped-GEMM timings at a
    fixed row count per expert can use it."""
    from mixture_experts_layer_59_b200 import synth
    for T, E, k in ((512, 16, 8), (96, 8, 4), (64, 64, 1)):
        cfg = synth.CONFIGS["coarse"].with_(T=T, d=64, f=64, E=E, k=k, routing="balanced")
        inp = synth.make_inputs(cfg, seed=0)
        _, idx, gate = O.route(None, None, k, logits_override=inp["logits_override"].numpy())
        assert all(len(set(r)) == k for r in idx.tolist())
        counts = np.bincount(idx.ravel(), minlength=E)
        assert (counts == T * k // E).all()
        np.testing.assert_allclose(gate.sum(axis=1), 1.0, rtol=0, atol=1e-12)
