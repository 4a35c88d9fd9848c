"""The compute ops of an expert-parallel step (mixture_experts_layer_59_b200.ep)
written with the CPU oracle, in float64 without bf16 staging, so that the
exchange and placement logic of ep.py can run on CPU ranks (gloo, or threads)
and be compared with the oracle's one-device layer on all ranks' tokens.

Test infrastructure: the package never imports this module."""
from __future__ import annotations

import numpy as np
import torch

from oracle import moe_oracle as O


def _np(t):
    return t.detach().cpu().numpy()


class OracleOps:
    def route(self, x, w_gate, k, logits_override=None):
        lo = None if logits_override is None else _np(logits_override).astype(np.float64)
        logits, idx, gate = O.route(_np(x), _np(w_gate), k, logits_override=lo)
        return torch.from_numpy(logits), torch.from_numpy(idx.astype(np.int64)), torch.from_numpy(gate)

    def permute(self, idx, gate, logits, E):
        p = O.exact_plan(_np(idx), _np(gate), E)
        return dict(np=p, offsets=torch.from_numpy(p["offsets"].astype(np.int32)),
                    row_token=torch.from_numpy(p["row_token"]),
                    row_gate=torch.from_numpy(p["row_gate"]),
                    slot_row=torch.from_numpy(p["slot_row"]))

    def gather_rows(self, src, plan, k):
        p = plan["np"]
        out = np.zeros((p["cap"], src.shape[1]))
        live = np.nonzero(p["row_token"] >= 0)[0]
        out[live] = _np(src)[p["row_token"][live]]
        return torch.from_numpy(out)

    def dispatch_counts(self, offsets):
        o = _np(offsets).astype(np.int64)
        return torch.from_numpy((o[1:] - o[:-1]).astype(np.int32))

    def receive_plan(self, recv_rows):
        # placement of the segment of (source s, local expert j): after every
        # earlier expert's rows, and after the earlier sources' rows of expert j
        r = _np(recv_rows).astype(np.int64)
        G, El = r.shape
        local_offsets = np.zeros(El + 1, np.int64)
        for j in range(El):
            local_offsets[j + 1] = local_offsets[j] + r[:, j].sum()
        recv_row = np.zeros((G, El), np.int64)
        for j in range(El):
            pos = local_offsets[j]
            for s in range(G):
                recv_row[s, j] = pos
                pos += r[s, j]
        return (torch.from_numpy(local_offsets.astype(np.int32)),
                torch.from_numpy(recv_row.astype(np.int32)))

    def expert_rows_fwd(self, xg, w1, w3, w2, offsets):
        xg, off = _np(xg), _np(offsets).astype(np.int64)
        f = w1.shape[2]
        H, Y = np.zeros((xg.shape[0], 2 * f)), np.zeros_like(xg)
        for j in range(len(off) - 1):
            lo, hi = off[j], off[j + 1]
            h1, h3, _, y = O.expert_rows_forward(xg[lo:hi], _np(w1[j]), _np(w3[j]), _np(w2[j]),
                                                 staged=False)
            H[lo:hi, :f], H[lo:hi, f:], Y[lo:hi] = h1, h3, y
        return torch.from_numpy(H), torch.from_numpy(Y)

    def combine(self, y_perm, plan, T, E, k):
        p, y = plan["np"], _np(y_perm)
        out = np.zeros((T, y.shape[1]))
        for t in range(T):
            for r in O.token_rows(p, t):
                out[t] += p["row_gate"][r] * y[r]
        return torch.from_numpy(out)

    def expert_rows_bwd(self, dog, xg, row_gate, H, w1, w3, w2, offsets):
        dog, xg, g, H = _np(dog), _np(xg), _np(row_gate), _np(H)
        off = _np(offsets).astype(np.int64)
        El, d, f = w1.shape
        dX, dS = np.zeros_like(xg), np.zeros(xg.shape[0])
        dw1, dw3, dw2 = np.zeros((El, d, f)), np.zeros((El, d, f)), np.zeros((El, f, d))
        for j in range(El):
            lo, hi = off[j], off[j + 1]
            ds, da1, da3, ga, dxp = O.expert_rows_backward(
                dog[lo:hi], g[lo:hi], H[lo:hi, :f], H[lo:hi, f:], _np(w1[j]), _np(w3[j]),
                _np(w2[j]), staged=False)
            dS[lo:hi], dX[lo:hi] = ds, dxp
            dw2[j] = ga.T @ dog[lo:hi]
            dw1[j] = xg[lo:hi].T @ da1
            dw3[j] = xg[lo:hi].T @ da3
        t = torch.from_numpy
        return dict(dX_rows=t(dX), dS=t(dS), dw1=t(dw1), dw3=t(dw3), dw2=t(dw2))

    def token_bwd(self, dx_rows, dS, x, w_gate, idx, gate, plan, router_grad):
        p, dxr, ds = plan["np"], _np(dx_rows), _np(dS)
        x, wg, idx, gate = _np(x), _np(w_gate), _np(idx), _np(gate)
        T, E = x.shape[0], wg.shape[1]
        dl, dx = np.zeros((T, E)), np.zeros_like(x)
        for t in range(T):
            rows = O.token_rows(p, t)
            dl[t] = O.token_router_grad(p, idx, gate, t, rows, ds[rows])
            for r in rows:
                dx[t] += dxr[r]
        dwg = np.zeros_like(wg)
        if router_grad:
            dx += dl @ wg.T
            dwg = x.T @ dl
        tt = torch.from_numpy
        return dict(dx=tt(dx), dw_gate=tt(dwg), dlogits=tt(dl))

    def check(self):
        pass


def make_problem(G, T, d, f, E, k, seed=0):
    """Per-rank tokens x_r, dout_r [T, d] and the shared weights (float64)."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((G * T, d))
    dout = rng.standard_normal((G * T, d))
    wg = rng.standard_normal((d, E)) / np.sqrt(d)
    w1 = rng.standard_normal((E, d, f)) / np.sqrt(d)
    w3 = rng.standard_normal((E, d, f)) / np.sqrt(d)
    w2 = rng.standard_normal((E, f, d)) / np.sqrt(f)
    return x, dout, wg, w1, w3, w2


def reference(x, dout, wg, w1, w3, w2, k):
    fwd = O.layer_fwd(x, wg, w1, w3, w2, k, staged=False)
    bwd = O.layer_bwd(dout, x, wg, w1, w3, w2, fwd, staged=False)
    return fwd, bwd


def run_rank(rank, exchange, G, T, d, f, E, k, seed=0):
    """One rank's forward + backward through ep.ExpertParallelMoE on the oracle ops."""
    from mixture_experts_layer_59_b200.ep import ExpertParallelMoE
    x, dout, wg, w1, w3, w2 = make_problem(G, T, d, f, E, k, seed)
    El = E // G
    sl, el = slice(rank * T, (rank + 1) * T), slice(rank * El, (rank + 1) * El)
    t = torch.from_numpy
    layer = ExpertParallelMoE(exchange, E, k, ops=OracleOps())
    out = layer.forward(t(x[sl]), t(wg), t(w1[el]), t(w3[el]), t(w2[el]))
    g = layer.backward(t(dout[sl]))
    return dict(out=out.numpy(), dx=g["dx"].numpy(), dw_gate=g["dw_gate"].numpy(),
                dlogits=g["dlogits"].numpy(), dw1=g["dw1"].numpy(), dw3=g["dw3"].numpy(),
                dw2=g["dw2"].numpy(), local_rows=layer.routing["local_rows"])
