"""CPU oracle for the token-choice MoE expert layer, forward and backward.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  It shares no code with the CUDA library and never imports it.

Everything is plain numpy in float64.  Each function restates one step of the
method as the source pages define it; a library primitive (matmul, argsort,
bincount) may serve as a step, with no blocking or fusion beyond that.

Sources (cited by page title and section):
  [Beam]     "From 501B to 23B: what is Beam doing" -- sec. 2.2 (router, top-k,
             weighted sum of experts), sec. 5.3 (MoELayer: top-k, then softmax
             of the k values, per-expert masked loop), sec. 5.4 (expert counts).
  [Trinity]  "Trinity Large: open 400B sparse MoE" commentary -- example 1
             (gate logits, torch.topk, softmax of the top-k), example 2
             (bincount of expert ids), example 3 (dispatch tokens into
             per-expert input lists, run experts, add outputs back per token).
  [SonicMoE] techwalker summary of SonicMoE -- sec. 1 (router-score gradient
             dS = <dA', A> instead of <dO, Y>; recompute instead of store),
             sec. 3 (token rounding: snap each expert's token count to the
             nearest multiple of the GEMM tile, e.g. 145 -> 128).
  [Olmo]     Olmo-core 3 news piece -- "row-wise expert parallelism puts data
             straight into expert input buffers", GPU-resident routing,
             grouped GEMM.
  [KJ]       "Breaking the hundred-billion-parameter barrier: how MoE reshapes
             distributed training" -- challenge 1, solution 1: load-balance
             loss L = lambda * CV(mean over the batch of G_i)^2.

Readings taken where the pages are silent:
  * top-k then softmax over the k selected logits (sec. 5.3 / example 1); ties
    in the logits go to the lowest expert id.
  * experts are SwiGLU: A = silu(x W1) * (x W3), Y = A W2.
  * rows of one expert are stored in ascending token order, and each expert's
    segment starts at a multiple of the tile (128 rows); padding rows are
    empty (token -1, weight 0).
  * bf16 "staging": in the bf16 path every tensor that is stored in bf16 or
    fed to a bf16 GEMM (H, A, Y, g*A, dH, dX_perm) is rounded to bf16
    (round-to-nearest-even) at the same point here; ``staged=False`` gives the
    ideal fp64 value.
  * token rounding: r_e = tile*round(c_e/tile) with halves rounding up, capped
    at tile*floor(T/tile); ranking key s_te = exp(l_te - LSE over the token's
    top-k logits); drops take the smallest keys (ties: larger token first),
    additions take the largest keys among unassigned tokens (ties: smaller
    token first); final weights are s_te without renormalisation.
  * noisy top-k gating ([Beam] sec. 3.3, second point: noise added to the
    routing scores in training): the caller draws the noise eps [T,E] and
    passes it in; routing (choice, gates, rounding scores) uses l + eps, and
    the gradient reaches the clean logits unchanged because eps depends on
    no parameter.
  * balance loss: G_i is token i's routing distribution over the E experts
    (its top-k gates, zeros elsewhere); CV is the population coefficient of
    variation over experts (std / mean); count statistics use the top-k
    choices before any rounding.

parity pins: tests/test_oracle_pins.py (brute force, dense masked evaluation,
closed-form 2-expert example, central finite differences, the 145 -> 128
rounding example, invariants, hand-derived values at every bf16 staging point; MXFP8 against torch's float8_e4m3fn conversion,
the 256-code table, closed-form scales and saturation).  No function here is
unpinned.
"""
from __future__ import annotations

import numpy as np

TILE = 128


# --------------------------------------------------------------------------
# elementary pieces
# --------------------------------------------------------------------------

def bf16_round(a):
    """Round float64 values to the nearest bfloat16 value (ties to even).

    bfloat16 keeps 8 significant bits and the float32 exponent range, so the
    spacing of representable values around |a| in [2^(e-1), 2^e) is 2^(e-8),
    and never finer than the subnormal spacing 2^-133.
    """
    a = np.asarray(a, dtype=np.float64)
    out = np.zeros_like(a)
    nz = a != 0
    if not np.any(nz):
        return out
    _, e = np.frexp(a[nz])                    # a = m * 2^e, 0.5 <= |m| < 1
    e = np.maximum(e, -125)
    ulp = np.ldexp(1.0, e - 8)
    out[nz] = np.rint(a[nz] / ulp) * ulp      # np.rint rounds halves to even
    return out


def _stage(a, staged):
    return bf16_round(a) if staged else a


def sigmoid(z):
    z = np.asarray(z, dtype=np.float64)
    return 0.5 * (1.0 + np.tanh(0.5 * z))


def silu(z):
    """silu(z) = z * sigmoid(z)."""
    return np.asarray(z, dtype=np.float64) * sigmoid(z)


def silu_grad(z):
    """d silu / dz = sigmoid(z) * (1 + z * (1 - sigmoid(z)))."""
    s = sigmoid(z)
    return s * (1.0 + z * (1.0 - s))


# --------------------------------------------------------------------------
# router: logits, top-k, softmax over the top-k  ([Beam] 2.2, 5.3; [Trinity] ex. 1)
# --------------------------------------------------------------------------

def route(x, w_gate, k, logits_override=None, logit_bias=None, gate_mode=0, logit_noise=None):
    """Router logits l = x W_gate (+ optional per-expert bias, + optional
    noise eps [T,E] drawn by the caller: noisy top-k gating, [Beam] 3.3), the
    k largest logits of each token (ties: lowest expert id first), and their
    gates:
    gate_mode 0: softmax over the k selected logits ([Beam] 5.3, [Trinity] ex. 1);
    gate_mode 1: softmax over all E logits, the k largest kept without
    renormalisation ([Beam] 2.2 formula, [Trinity] challenge 1).

    Returns (logits [T,E] f64, idx [T,k] int32, gate [T,k] f64).
    """
    if logits_override is not None:
        logits = np.array(logits_override, dtype=np.float64)
    else:
        logits = np.asarray(x, np.float64) @ np.asarray(w_gate, np.float64)
    if logit_bias is not None:
        logits = logits + np.asarray(logit_bias, np.float64)[None, :]
    if logit_noise is not None:
        logits = logits + np.asarray(logit_noise, np.float64)
    # a stable sort of the negated logits keeps equal values in ascending id
    idx = np.argsort(-logits, axis=1, kind="stable")[:, :k]
    top = np.take_along_axis(logits, idx, axis=1)
    if gate_mode == 0:
        ex = np.exp(top - top[:, :1])
        gate = ex / ex.sum(axis=1, keepdims=True)
    else:
        m = logits.max(axis=1, keepdims=True)
        z = np.exp(logits - m).sum(axis=1, keepdims=True)
        gate = np.exp(top - m) / z
    return logits, idx.astype(np.int32), gate


# --------------------------------------------------------------------------
# permutation into expert-contiguous rows  ([Trinity] ex. 2-3; [Olmo]; [Beam] 5.4)
# --------------------------------------------------------------------------

def _pad(n, tile):
    return ((n + tile - 1) // tile) * tile


def row_capacity(T, E, k, tile=TILE):
    """Rows any plan may occupy: every slot plus a tile of slack per expert."""
    return T * k + E * tile


def exact_plan(idx, gate, E, tile=TILE):
    """Dropless permutation.  counts[e] = number of tokens that chose e;
    expert e owns rows [offsets[e], offsets[e] + counts[e]) in ascending token
    order; offsets are the exclusive prefix sum of counts padded to the tile.
    """
    idx = np.asarray(idx)
    T, k = idx.shape
    cap = row_capacity(T, E, k, tile)
    counts = np.bincount(idx.ravel(), minlength=E).astype(np.int64)
    offsets = np.zeros(E + 1, np.int64)
    offsets[1:] = np.cumsum(_pad(counts, tile))
    row_token = np.full(cap, -1, np.int64)
    row_slot = np.full(cap, -1, np.int64)
    row_gate = np.zeros(cap, np.float64)
    slot_row = np.full(T * k, -1, np.int64)
    flat = idx.ravel()
    # slots are numbered token-major (s = t*k + j); a stable sort by expert
    # keeps ascending token order inside each expert
    order = np.argsort(flat, kind="stable")
    start = np.zeros(E + 1, np.int64)
    start[1:] = np.cumsum(counts)
    for e in range(E):
        slots = order[start[e]:start[e + 1]]
        rows = offsets[e] + np.arange(len(slots))
        row_token[rows] = slots // k
        row_slot[rows] = slots
        row_gate[rows] = np.asarray(gate, np.float64).ravel()[slots]
        slot_row[slots] = rows
    return dict(mode="exact", T=T, E=E, k=k, tile=tile, cap=cap, counts=counts,
                offsets=offsets, row_token=row_token, row_slot=row_slot,
                row_gate=row_gate, slot_row=slot_row, extra_row=None,
                R=int(offsets[-1]))


def rounded_target(counts, T, tile=TILE):
    """Token rounding target ([SonicMoE] sec. 3): the multiple of the tile
    nearest to each count (an exact half rounds up), capped at the largest
    multiple of the tile that does not exceed T."""
    counts = np.asarray(counts, np.int64)
    r = tile * ((counts + tile // 2) // tile)
    return np.minimum(r, tile * (T // tile))


def rounding_keys(logits, idx, gate_mode=0):
    """Log-domain ranking key of every (token, expert) pair: the log of the
    weight the pair has (or would have) as a routed pair, i.e.
    l_te - LSE over the token's top-k logits (gate_mode 0) or over all E
    logits (gate_mode 1)."""
    logits = np.asarray(logits, np.float64)
    if gate_mode == 0:
        top = np.take_along_axis(logits, np.asarray(idx), axis=1)
    else:
        top = logits
    m = top.max(axis=1)
    lse = m + np.log(np.exp(top - m[:, None]).sum(axis=1))
    return logits - lse[:, None]


def capacity_target(counts, capacity):
    """Capacity factor ([Beam] sec. 2.3): at most `capacity` tokens per expert."""
    return np.minimum(np.asarray(counts, np.int64), capacity)


def rounded_plan(idx, logits, E, tile=TILE, gate_mode=0, capacity=None):
    """Token-rounded permutation ([SonicMoE] sec. 3 with the readings in the
    module docstring), or with ``capacity`` the capacity-factor permutation
    ([Beam] sec. 2.3: experts above capacity drop their lowest-scoring pairs,
    ties dropping the larger token first; no pairs are added; segments are
    padded to the tile).  Adds ``extra_row[T,E]`` (row of an added pair, else
    -1) and ``dropped``/``added`` masks for checking."""
    idx = np.asarray(idx)
    T, k = idx.shape
    cap = row_capacity(T, E, k, tile)
    counts = np.bincount(idx.ravel(), minlength=E).astype(np.int64)
    if capacity is None:
        target = rounded_target(counts, T, tile)
    else:
        target = capacity_target(counts, capacity)
    key = rounding_keys(logits, idx, gate_mode)
    assigned = np.zeros((T, E), bool)
    assigned[np.arange(T)[:, None], idx] = True
    final = assigned.copy()
    toks = np.arange(T)
    for e in range(E):
        if target[e] < counts[e]:
            cand = toks[assigned[:, e]]
            # order by key descending, then token ascending; keep the first r_e
            order = cand[np.lexsort((cand, -key[cand, e]))]
            final[order[target[e]:], e] = False
        elif target[e] > counts[e]:
            cand = toks[~assigned[:, e]]
            order = cand[np.lexsort((cand, -key[cand, e]))]
            final[order[:target[e] - counts[e]], e] = True
    offsets = np.zeros(E + 1, np.int64)
    offsets[1:] = np.cumsum(_pad(target, tile))
    row_token = np.full(cap, -1, np.int64)
    row_slot = np.full(cap, -1, np.int64)
    row_gate = np.zeros(cap, np.float64)
    slot_row = np.full(T * k, -1, np.int64)
    extra_row = np.full((T, E), -1, np.int64)
    slot_of = np.full((T, E), -1, np.int64)
    slot_of[np.arange(T)[:, None], idx] = np.arange(T * k).reshape(T, k)
    for e in range(E):
        members = toks[final[:, e]]
        rows = offsets[e] + np.arange(len(members))
        row_token[rows] = members
        row_gate[rows] = np.exp(key[members, e])
        s = slot_of[members, e]
        row_slot[rows] = s
        kept = s >= 0
        slot_row[s[kept]] = rows[kept]
        extra_row[members[~kept], e] = rows[~kept]
    return dict(mode="rounded" if capacity is None else "capacity", T=T, E=E, k=k, tile=tile,
                cap=cap, counts=counts, target=target, offsets=offsets, row_token=row_token,
                row_slot=row_slot, row_gate=row_gate, slot_row=slot_row,
                extra_row=extra_row if capacity is None else None, dropped=assigned & ~final,
                added=final & ~assigned, R=int(offsets[-1]), key=key, gate_mode=gate_mode)


def token_rows(plan, t):
    """All rows of token t: its kept slots in slot order, then the rows added
    by token rounding in ascending expert order."""
    k = plan["k"]
    rows = [int(r) for r in plan["slot_row"][t * k:(t + 1) * k] if r >= 0]
    if plan["extra_row"] is not None:
        rows += [int(r) for r in plan["extra_row"][t] if r >= 0]
    return rows


def row_expert(plan, rows):
    """Expert owning each row (the segment the row falls in)."""
    return np.searchsorted(plan["offsets"], np.asarray(rows), side="right") - 1


# --------------------------------------------------------------------------
# MXFP8: the OCP Microscaling (MX) v1.0 format with E4M3 elements -- blocks of
# 32 consecutive elements share one power-of-two scale X = 2^e (an E8M0 code
# e + 127).  The pages name the format (Olmo-core 3 news piece: "MXFP8
# low-precision switch"; SonicMoE summary, future work) without defining it;
# this is the public definition.  Blocks run along the contraction dimension
# of each GEMM, the only direction in which the scales factor out of a dot
# product.
# --------------------------------------------------------------------------
MX_BLOCK = 32
E4M3_MAX = 448.0       # 1.75 * 2^8, the largest finite E4M3 value
E4M3_EMAX = 8          # exponent of that value
E4M3_EMIN = -6         # exponent of the smallest normal value


def e4m3_round(v):
    """Nearest E4M3 value (ties to the even mantissa), saturated to +-448.

    A value of binade 2^e (e >= -6) is rounded on the grid 2^(e-3) (three
    mantissa bits); below 2^-6 the grid is the subnormal step 2^-9."""
    v = np.asarray(v, np.float64)
    a = np.abs(v)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))       # a = m 2^ex, m in [0.5, 1)
    e = np.maximum(ex - 1, E4M3_EMIN)
    step = np.ldexp(1.0, e - 3)
    q = np.minimum(np.round(a / step) * step, E4M3_MAX)   # np.round: half to even
    return np.where(np.signbit(v), -q, q)


def e4m3_encode(q):
    """uint8 codes of values already on the E4M3 grid (sign, 4-bit exponent
    with bias 7, 3-bit mantissa; -0 keeps its sign bit)."""
    q = np.asarray(q, np.float64)
    a = np.abs(q)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))
    e = ex - 1
    normal = (a > 0) & (e >= E4M3_EMIN)
    exp_field = np.where(normal, e + 7, 0)
    mant = np.where(normal, a / np.ldexp(1.0, e) - 1.0, a / 2.0 ** -9) * np.where(normal, 8, 1)
    code = (exp_field.astype(np.int64) << 3) | np.rint(mant).astype(np.int64)
    return (code | (np.signbit(q).astype(np.int64) << 7)).astype(np.uint8)


def e4m3_decode(code):
    """Values of uint8 E4M3 codes (0x7F and 0xFF are NaN)."""
    c = np.asarray(code, np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    ef, mf = (c >> 3) & 0xF, c & 7
    val = np.where(ef == 0, mf * 2.0 ** -9, (1.0 + mf / 8.0) * np.ldexp(1.0, ef - 7))
    return np.where((c & 0x7F) == 0x7F, np.nan, sign * val)


def mx_shared_exp(amax):
    """Shared exponent of a block: floor(log2 amax) - 8 (so that the block's
    largest element lands in [256, 512) before rounding), clamped to the E8M0
    range [-127, 127]; -127 for an all-zero block."""
    amax = np.asarray(amax, np.float64)
    _, ex = np.frexp(np.where(amax > 0, amax, 1.0))
    return np.where(amax > 0, np.clip(ex - 1 - E4M3_EMAX, -127, 127), -127).astype(np.int64)


def mx_quantize(a, axis):
    """MXFP8 quantisation of ``a`` in blocks of 32 along ``axis``.

    Returns (q, se): q the E4M3 element values (on the E4M3 grid, shape of
    ``a``) and se the shared exponents (one per block, the block axis in place
    of ``axis``); the represented value is q * 2^se."""
    a = np.moveaxis(np.asarray(a, np.float64), axis, -1)
    n = a.shape[-1]
    assert n % MX_BLOCK == 0
    blk = a.reshape(a.shape[:-1] + (n // MX_BLOCK, MX_BLOCK))
    se = mx_shared_exp(np.abs(blk).max(axis=-1))
    q = e4m3_round(blk / np.ldexp(1.0, se)[..., None])
    return (np.moveaxis(q.reshape(a.shape), -1, axis), np.moveaxis(se, -1, axis))


def mx_dequantize(q, se, axis):
    q = np.moveaxis(np.asarray(q, np.float64), axis, -1)
    se = np.moveaxis(np.asarray(se), axis, -1)
    x = q * np.repeat(np.ldexp(1.0, se), MX_BLOCK, axis=-1)
    return np.moveaxis(x, -1, axis)


def mx_fake_quant(a, axis):
    """The values MXFP8 represents for ``a`` (blocks of 32 along ``axis``)."""
    return mx_dequantize(*mx_quantize(a, axis), axis)


# --------------------------------------------------------------------------
# expert SwiGLU FFN on the rows of one expert
# --------------------------------------------------------------------------

def expert_rows_forward(xr, w1e, w3e, w2e, staged, precision="bf16"):
    """H = [x W1 | x W3] (bf16-staged if ``staged``), A = silu(h1) * h3,
    Y = A W2, for the rows ``xr`` [n,d] routed to one expert.

    precision "mxfp8": both GEMMs take MXFP8 operands -- x and W1/W3 in blocks
    along d, A (after its bf16 staging) and W2 in blocks along f -- with exact
    products and sums of the represented values."""
    xr = np.asarray(xr, np.float64)
    if precision == "mxfp8":
        xq = mx_fake_quant(xr, 1)
        h1 = _stage(xq @ mx_fake_quant(w1e, 0), staged)
        h3 = _stage(xq @ mx_fake_quant(w3e, 0), staged)
        a = _stage(silu(h1) * h3, staged)
        y = _stage(mx_fake_quant(a, 1) @ mx_fake_quant(w2e, 0), staged)
        return h1, h3, a, y
    h1 = _stage(xr @ w1e, staged)
    h3 = _stage(xr @ w3e, staged)
    a = _stage(silu(h1) * h3, staged)
    y = _stage(a @ w2e, staged)
    return h1, h3, a, y


def expert_rows_backward(dor, gr, h1, h3, w1e, w3e, w2e, staged, precision="bf16"):
    """Backward of one expert's rows given dO rows ``dor`` and row weights ``gr``.

    dA' = dO W2^T                       (gradient of A before gate scaling)
    dS  = <dA', A>                      ([SonicMoE] sec. 1: no stored Y needed)
    dA  = g dA';  da3 = dA silu(h1);  da1 = dA h3 silu'(h1)
    g*A (operand of dW2), dX_perm = da1 W1^T + da3 W3^T.

    precision "mxfp8": the dX_perm GEMM takes MXFP8 operands -- dH (after its
    bf16 staging) and W1, W3, all in blocks along f; the other GEMMs keep the
    unquantised operands.
    """
    dor = np.asarray(dor, np.float64)
    a = _stage(silu(h1) * h3, staged)
    dap = dor @ w2e.T
    ds = np.sum(dap * a, axis=1)
    da = gr[:, None] * dap
    da3 = _stage(da * silu(h1), staged)
    da1 = _stage(da * h3 * silu_grad(h1), staged)
    ga = _stage(gr[:, None] * a, staged)
    if precision == "mxfp8":
        dxp = _stage(mx_fake_quant(da1, 1) @ mx_fake_quant(w1e, 1).T
                     + mx_fake_quant(da3, 1) @ mx_fake_quant(w3e, 1).T, staged)
    else:
        dxp = _stage(da1 @ w1e.T + da3 @ w3e.T, staged)
    return ds, da1, da3, ga, dxp


# --------------------------------------------------------------------------
# full layer, and the same quantities on a subset of tokens / experts
# --------------------------------------------------------------------------

def _f64(a):
    return np.asarray(a, dtype=np.float64)


def rows_compute(rows, plan, x, w1, w3, w2, dout=None, staged=True, precision="bf16"):
    """Forward (and, given dout, backward) quantities of the listed rows.

    With precision "mxfp8" the forward GEMMs and the backward dX_perm GEMM
    take MXFP8 operands; the backward uses that forward's H, and the gradients
    pass the quantisers straight through (the other backward GEMMs use the
    unquantised x, weights and staged intermediates).

    Rows are grouped by the expert that owns them; padding rows give zeros.
    w1, w3, w2 may be arrays or any object whose [e] gives expert e's matrix
    (weights are read one expert at a time).
    Returns a dict of arrays aligned with ``rows``: H [n,2f], A [n,f],
    Y [n,d] and, with dout, dS [n], dH [n,2f], gA [n,f], dXp [n,d].
    """
    rows = np.asarray(rows, np.int64)
    x = _f64(x)
    n, d, f = len(rows), x.shape[1], np.shape(w1[0])[1]
    res = dict(H=np.zeros((n, 2 * f)), A=np.zeros((n, f)), Y=np.zeros((n, d)))
    if dout is not None:
        dout = _f64(dout)
        res.update(dS=np.zeros(n), dH=np.zeros((n, 2 * f)), gA=np.zeros((n, f)),
                   dXp=np.zeros((n, d)))
    toks_all = plan["row_token"][rows]
    es = row_expert(plan, rows)
    for e in np.unique(es[toks_all >= 0]):
        sel = np.nonzero((es == e) & (toks_all >= 0))[0]
        toks = toks_all[sel]
        w1e, w3e, w2e = _f64(w1[e]), _f64(w3[e]), _f64(w2[e])
        h1, h3, a, y = expert_rows_forward(x[toks], w1e, w3e, w2e, staged, precision)
        res["H"][sel, :f], res["H"][sel, f:], res["A"][sel], res["Y"][sel] = h1, h3, a, y
        if dout is not None:
            g = plan["row_gate"][rows[sel]]
            ds, da1, da3, ga, dxp = expert_rows_backward(
                dout[toks], g, h1, h3, w1e, w3e, w2e, staged, precision)
            res["dS"][sel] = ds
            res["dH"][sel, :f], res["dH"][sel, f:] = da1, da3
            res["gA"][sel] = ga
            res["dXp"][sel] = dxp
    return res


def token_router_grad(plan, idx, gate, t, rows, dS_rows, logits=None):
    """dlogits of token t from the router-score gradients of its rows.

    F_t: the final rows of token t with weights s; K_t: its top-k experts.
    gate_mode 0 (p = softmax over K_t):
        dl_te = [e in F_t] s_te dS_te - [e in K_t] p_te * sum_{e' in F_t} s_te' dS_te'.
    gate_mode 1 (p = softmax over all E, s_te = p_te):
        dl_te = [e in F_t] p_te dS_te - p_te * sum_{e' in F_t} p_te' dS_te'   (every e).
    For the dropless plan and gate_mode 0 this is g_e (dS_e - sum g dS).
    """
    E, k = plan["E"], plan["k"]
    mode = plan.get("gate_mode", 0)
    dl = np.zeros(E)
    tot = 0.0
    for r, ds, e in zip(rows, dS_rows, row_expert(plan, rows)):
        v = plan["row_gate"][r] * ds
        dl[e] += v
        tot += v
    if mode == 0:
        for j in range(k):
            dl[idx[t, j]] -= gate[t, j] * tot
    else:
        lt = np.asarray(logits[t], np.float64)
        p = np.exp(lt - lt.max())
        p /= p.sum()
        dl -= p * tot
    return dl


def make_plan(idx, gate, logits, E, tile=TILE, round_mode=0, gate_mode=0, capacity=None):
    """round_mode 0: dropless; 1: token rounding; 2: capacity factor."""
    if round_mode == 0:
        plan = exact_plan(idx, gate, E, tile)
        plan["gate_mode"] = gate_mode
        return plan
    if round_mode == 1:
        return rounded_plan(idx, logits, E, tile, gate_mode)
    return rounded_plan(idx, logits, E, tile, gate_mode, capacity=capacity)


def layer_fwd(x, w_gate, w1, w3, w2, k, tile=TILE, round_mode=0,
              logits_override=None, logit_bias=None, staged=True, gate_mode=0, capacity=None,
              logit_noise=None, precision="bf16"):
    """Full forward: route, permute, expert FFN on every row, combine.
    precision "mxfp8": the expert GEMMs take MXFP8 operands (expert_rows_forward)."""
    logits, idx, gate = route(x, w_gate, k, logits_override, logit_bias, gate_mode, logit_noise)
    T, E = logits.shape
    plan = make_plan(idx, gate, logits, E, tile, round_mode, gate_mode, capacity)
    rows = np.arange(plan["R"])
    res = rows_compute(rows, plan, x, w1, w3, w2, None, staged, precision)
    out = np.zeros((T, np.shape(x)[1]))
    for t in range(T):
        for r in token_rows(plan, t):
            out[t] += plan["row_gate"][r] * res["Y"][r]
    return dict(logits=logits, idx=idx, gate=gate, plan=plan, H=res["H"],
                A=res["A"], Y=res["Y"], out=out, precision=precision)


def _segment(live_vals, live, width):
    """An expert's segment of the row space as a dense [rows, width] matrix:
    the live rows' values in row order, zeros in the padding rows."""
    out = np.zeros((len(live), width))
    out[live] = live_vals
    return out


def mx_wgrad(a_seg, b_seg):
    """Weight gradient of one expert on MXFP8 operands: a^T b with both
    operands quantised along the token axis -- the contraction dimension of
    this GEMM -- in blocks of 32 consecutive rows of the expert's segment of
    the row space (padding rows are zero rows of the segment)."""
    return mx_fake_quant(a_seg, 0).T @ mx_fake_quant(b_seg, 0)


def layer_bwd(dout, x, w_gate, w1, w3, w2, fwd, staged=True, router_grad_on=True,
              extra_dlogits=None, mx_wgrad_on=False):
    """Full backward from the saved set {x, logits, idx, gate, plan, H}.

    dW2_e = sum_rows (g A)^T dO,  [dW1|dW3]_e = sum_rows x^T dH,
    dx_t = sum over the rows of t of dX_perm + dlogits_t W_gate^T,
    dW_gate = x^T dlogits.  Returns dx, dw_gate, dw1, dw3, dw2, dS [R], dlogits.
    mx_wgrad_on: the weight-gradient GEMMs take MXFP8 operands (mx_wgrad) over
    each expert's whole segment, padding rows included.
    """
    dout, x, w_gate, w1, w3, w2 = map(_f64, (dout, x, w_gate, w1, w3, w2))
    plan = fwd["plan"]
    T, d = x.shape
    E, _, f = w1.shape
    R = plan["R"]
    rows = np.arange(R)
    res = rows_compute(rows, plan, x, w1, w3, w2, dout, staged, fwd.get("precision", "bf16"))
    dw1, dw3, dw2 = np.zeros_like(w1), np.zeros_like(w3), np.zeros_like(w2)
    for e in range(E):
        lo, hi = plan["offsets"][e], plan["offsets"][e + 1]
        toks = plan["row_token"][lo:hi]
        live = toks >= 0
        r = np.arange(lo, hi)[live]
        if mx_wgrad_on:
            seg = lambda rows_val, width: _segment(rows_val, live, width)
            dw2[e] = mx_wgrad(seg(res["gA"][r], f), seg(dout[toks[live]], d))
            dw13 = mx_wgrad(seg(x[toks[live]], d), seg(res["dH"][r], 2 * f))
            dw1[e], dw3[e] = dw13[:, :f], dw13[:, f:]
            continue
        dw2[e] = res["gA"][r].T @ dout[toks[live]]
        dw1[e] = x[toks[live]].T @ res["dH"][r, :f]
        dw3[e] = x[toks[live]].T @ res["dH"][r, f:]
    dlogits = np.zeros((T, E))
    dx = np.zeros((T, d))
    for t in range(T):
        tr = token_rows(plan, t)
        dlogits[t] = token_router_grad(plan, fwd["idx"], fwd["gate"], t, tr, res["dS"][tr],
                                       fwd["logits"])
        for r in tr:
            dx[t] += res["dXp"][r]
    if extra_dlogits is not None:      # gradient of auxiliary router losses
        dlogits = dlogits + np.asarray(extra_dlogits, np.float64)
    dw_gate = np.zeros((d, E))
    if router_grad_on:
        dx += dlogits @ w_gate.T
        dw_gate = x.T @ dlogits
    return dict(dx=dx, dw_gate=dw_gate, dw1=dw1, dw3=dw3, dw2=dw2, dS=res["dS"],
                dlogits=dlogits, dXp=res["dXp"], dH=res["dH"])


def sampled_tokens(tokens, dout, x, w_gate, w1, w3, w2, fwd, staged=True, router_grad_on=True):
    """out, dx, dlogits and per-row dS for a subset of tokens only.  Each of
    these depends on nothing but the token itself and its experts' weights,
    so the values equal those of the full layer."""
    plan = fwd["plan"]
    dout, x, w_gate = _f64(dout), _f64(x), _f64(w_gate)
    per_tok = [token_rows(plan, t) for t in tokens]
    all_rows = [r for tr in per_tok for r in tr]
    res = rows_compute(all_rows, plan, x, w1, w3, w2, dout, staged, fwd.get("precision", "bf16"))
    out, dx, dl, dS = {}, {}, {}, {}
    pos = 0
    for t, tr in zip(tokens, per_tok):
        sl = slice(pos, pos + len(tr))
        pos += len(tr)
        out[t] = (plan["row_gate"][tr][:, None] * res["Y"][sl]).sum(axis=0)
        dl[t] = token_router_grad(plan, fwd["idx"], fwd["gate"], t, tr, res["dS"][sl],
                                  fwd["logits"])
        dx[t] = res["dXp"][sl].sum(axis=0)
        if router_grad_on:
            dx[t] = dx[t] + dl[t] @ w_gate.T
        for r, v in zip(tr, res["dS"][sl]):
            dS[r] = v
    return dict(out=out, dx=dx, dlogits=dl, dS=dS)


def sampled_expert_grads(experts, dout, x, w1, w3, w2, fwd, staged=True):
    """dW1, dW3, dW2 of the listed experts (sums over that expert's rows)."""
    plan = fwd["plan"]
    dout, x = _f64(dout), _f64(x)
    f = np.shape(w1[0])[1]
    out = {}
    for e in experts:
        lo, hi = plan["offsets"][e], plan["offsets"][e + 1]
        toks = plan["row_token"][lo:hi]
        live = toks >= 0
        rows = np.arange(lo, hi)[live]
        res = rows_compute(rows, plan, x, w1, w3, w2, dout, staged, fwd.get("precision", "bf16"))
        tk = toks[live]
        out[e] = dict(dw2=res["gA"].T @ dout[tk], dw1=x[tk].T @ res["dH"][:, :f],
                      dw3=x[tk].T @ res["dH"][:, f:])
    return out


def expert_grad_slices(e, cols, dout, x, w1e, w3e, w2e, fwd, staged=True):
    """Selected columns of dW1_e and dW3_e (all d rows) and the same-numbered
    rows of dW2_e (all d columns), from expert e's rows.

    Column c of H1/H3/A/dH involves only column c of W1_e, W3_e and row c of
    W2_e, so these slices follow from the per-element formulas of
    expert_rows_forward / expert_rows_backward restricted to those columns.
    """
    plan = fwd["plan"]
    dout, x = _f64(dout), _f64(x)
    cols = np.asarray(cols)
    lo, hi = plan["offsets"][e], plan["offsets"][e + 1]
    toks = plan["row_token"][lo:hi]
    live = toks >= 0
    tk = toks[live]
    g = plan["row_gate"][lo:hi][live]
    xr, dor = x[tk], dout[tk]
    w1c, w3c, w2r = _f64(w1e)[:, cols], _f64(w3e)[:, cols], _f64(w2e)[cols, :]
    if fwd.get("precision", "bf16") == "mxfp8":
        # H from MXFP8 operands (blocks along d: columns quantise independently)
        xq = mx_fake_quant(xr, 1)
        h1 = _stage(xq @ mx_fake_quant(w1c, 0), staged)
        h3 = _stage(xq @ mx_fake_quant(w3c, 0), staged)
    else:
        h1 = _stage(xr @ w1c, staged)
        h3 = _stage(xr @ w3c, staged)
    a = _stage(silu(h1) * h3, staged)
    dap = dor @ w2r.T
    da = g[:, None] * dap
    da3 = _stage(da * silu(h1), staged)
    da1 = _stage(da * h3 * silu_grad(h1), staged)
    ga = _stage(g[:, None] * a, staged)
    return dict(dw1=xr.T @ da1, dw3=xr.T @ da3, dw2=ga.T @ dor)


# --------------------------------------------------------------------------
# load-balance loss and routing statistics  ([KJ] challenge 1; [Trinity]
# example 2; [Beam] sec. 2.3 / 5.4)
# --------------------------------------------------------------------------

def balance_loss(idx, gate, E, lam):
    """L = lam * CV(importance)^2 with importance_e = mean over tokens of the
    token's routing weight on expert e (0 if e is not among its top-k).

    Returns dict(loss, importance [E], dgate [T,k] = dL/dgate, counts [E],
    max_share, count_cv2, count_mse) where the count statistics follow the
    per-expert token histogram: max share of all assignments, CV^2 of the
    counts and the mean squared deviation of the counts from their mean.
    """
    idx = np.asarray(idx)
    gate = np.asarray(gate, np.float64)
    T, k = idx.shape
    G = np.zeros((T, E))
    G[np.arange(T)[:, None], idx] = gate
    imp = G.mean(axis=0)
    m = imp.mean()
    var = ((imp - m) ** 2).mean()
    loss = lam * var / m ** 2
    # d(var/m^2)/d imp_e = (2/E)(imp_e - m)/m^2 - 2 var/(E m^3)
    dimp = lam * (2.0 / E * (imp - m) / m ** 2 - 2.0 * var / (E * m ** 3))
    dgate = dimp[idx] / T
    counts = np.bincount(idx.ravel(), minlength=E).astype(np.float64)
    cm = counts.mean()
    return dict(loss=loss, importance=imp, dgate=dgate, counts=counts,
                max_share=counts.max() / counts.sum(),
                count_cv2=((counts - cm) ** 2).mean() / cm ** 2,
                count_mse=((counts - cm) ** 2).mean())


def gate_grad_to_logits(idx, gate, dgate, E, gate_mode=0, logits=None):
    """dlogits from a gradient a = dgate on the top-k gates:
    gate_mode 0: dl_t,idx_j = g_j (a_j - sum_i g_i a_i), zero elsewhere;
    gate_mode 1: dl_te = [e in K_t] p_e a_e - p_e sum_i g_i a_i (every e)."""
    idx = np.asarray(idx)
    gate = np.asarray(gate, np.float64)
    dgate = np.asarray(dgate, np.float64)
    T, k = idx.shape
    dl = np.zeros((T, E))
    tot = (gate * dgate).sum(axis=1, keepdims=True)
    if gate_mode == 0:
        dl[np.arange(T)[:, None], idx] = gate * (dgate - tot)
    else:
        lg = np.asarray(logits, np.float64)
        p = np.exp(lg - lg.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        dl = -p * tot
        dl[np.arange(T)[:, None], idx] += gate * dgate
    return dl
