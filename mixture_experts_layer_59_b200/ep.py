"""Expert parallelism: the MoE layer over G ranks, each owning E/G experts.

The Olmo-core 3 news piece keeps experts resident on their GPU and routes the
data to them ("row-wise expert parallelism places rows straight into the
experts' input buffers"); the Beam article (sec. 4.2) describes the same
split with an all-to-all exchange of tokens.  Here rank g owns experts
g*El .. g*El+El-1 (El = E/G).  One step on every rank:

forward
  1. route, permute and gather this rank's tokens into its row space (the
     library's kernels, as on one GPU); the segments of rank g's experts
     are contiguous rows, so the row space itself is the send buffer;
  2. exchange the segment lengths (moe_ep_dispatch_counts -> all-to-all of
     E/G counts per peer) and place the incoming segments
     (moe_ep_receive_plan); the placement table comes to the host once,
     because the transfers need their sizes there;
  3. send the gathered rows and their weights to the experts' ranks;
  4. grouped GEMMs on the received rows (moe_expert_rows_fwd);
  5. return Y rows to the tokens' ranks, then combine (moe_combine).
backward
  6. gather dO rows, send them like the x rows;
  7. expert side (moe_expert_rows_bwd): dS, dX rows and the weight
     gradients of the local experts, complete because every row of a local
     expert is here;
  8. return dX rows and dS, then the token side (moe_token_bwd): dlogits,
     dx and this rank's share of dW_gate, summed over ranks (the router is
     replicated, data-parallel).

Every segment moves whole (128-aligned, padding rows included), so received
rows keep the tile alignment the grouped GEMMs need; with token rounding the
segments have no padding at all.  Every rank makes the same collective calls
in the same order.  The exchange is pluggable: ``TorchDistExchange`` uses
torch.distributed (NCCL send/recv between GPUs, gloo on CPU);
``LocalGroup`` runs G ranks as threads of one process that copy rows
between each other (G ranks on one device, for tests).  The compute ops are
pluggable too (``CudaOps``: the library's kernels; there is no other
implementation in the package).
"""
from __future__ import annotations

import threading

import torch

from . import binding as B


class CudaOps:
    """The per-rank compute of an expert-parallel step: the library's calls."""

    def route(self, x, w_gate, k, logits_override=None):
        return B.moe_route(x, w_gate, k, logits_override=logits_override,
                           T=x.shape[0], E=w_gate.shape[1])

    def permute(self, idx, gate, logits, E):
        return B.moe_permute(idx, gate, logits, E, B.MOE_ROUND_NONE)

    def gather_rows(self, src, plan, k):
        return B.moe_gather_rows(src, plan, k)

    def dispatch_counts(self, offsets):
        return B.moe_ep_dispatch_counts(offsets)

    def receive_plan(self, recv_rows):
        return B.moe_ep_receive_plan(recv_rows)

    def expert_rows_fwd(self, xg, w1, w3, w2, offsets):
        return B.moe_expert_rows_fwd(xg, w1, w3, w2, offsets)

    def combine(self, y_perm, plan, T, E, k):
        return B.moe_combine(y_perm, plan["row_gate"], plan["slot_row"], plan.get("extra_row"),
                             T, E, k)

    def expert_rows_bwd(self, dog, xg, row_gate, H, w1, w3, w2, offsets):
        return B.moe_expert_rows_bwd(dog, xg, row_gate, H, w1, w3, w2, offsets)

    def token_bwd(self, dx_rows, dS, x, w_gate, idx, gate, plan, router_grad):
        return B.moe_token_bwd(dx_rows, dS, x, w_gate, idx, gate, plan, router_grad=router_grad)

    def check(self):
        B.moe_check_status()


# ------------------------------------------------------------------ exchanges
class TorchDistExchange:
    """Collectives of the step over the default torch.distributed group."""

    def __init__(self):
        import torch.distributed as dist
        self.dist = dist
        self.rank = dist.get_rank()
        self.world = dist.get_world_size()

    def all_to_all_counts(self, send, el):
        """recv[s*el + j] = send_s[rank*el + j] for every source rank s."""
        recv = torch.empty_like(send)
        self.dist.all_to_all_single(recv, send)
        return recv

    def move(self, src, dst, sends, recvs):
        """sends: (peer, tag, first row, rows) blocks of ``src`` for each peer;
        recvs: (peer, tag, first row, rows) blocks of ``dst`` from each peer.
        Blocks of one peer pair are matched in order (and by tag)."""
        ops = []
        own = {}
        for p, j, off, n in sends:
            if p == self.rank:
                own[j] = src[off:off + n]
            else:
                ops.append(self.dist.P2POp(self.dist.isend, src[off:off + n].contiguous(), p, tag=j))
        for p, j, off, n in recvs:
            if p == self.rank:
                dst[off:off + n].copy_(own[j])
            else:
                ops.append(self.dist.P2POp(self.dist.irecv, dst[off:off + n], p, tag=j))
        if ops:
            for w in self.dist.batch_isend_irecv(ops):
                w.wait()

    def all_reduce_sum(self, t):
        self.dist.all_reduce(t, op=self.dist.ReduceOp.SUM)
        return t


class LocalGroup:
    """G ranks as threads of one process: each rank's exchange copies rows
    straight from the other ranks' tensors.  Every call is a barrier, so a
    rank that raises breaks the barrier of the others (after ``timeout``
    seconds at most) instead of leaving them waiting."""

    def __init__(self, world, timeout=120.0):
        self.world = world
        self.barrier = threading.Barrier(world, timeout=timeout)
        self.slots = {}

    def member(self, rank):
        return _LocalExchange(self, rank)

    def run(self, fn):
        """Run fn(rank, exchange) on every rank in its own thread; returns the
        results by rank, re-raising the first exception."""
        res, errs = [None] * self.world, [None] * self.world

        def body(r):
            try:
                res[r] = fn(r, self.member(r))
            except BaseException as e:  # noqa: BLE001 -- re-raised below
                errs[r] = e
                self.barrier.abort()

        th = [threading.Thread(target=body, args=(r,)) for r in range(self.world)]
        for t in th:
            t.start()
        for t in th:
            t.join()
        for e in errs:
            if e is not None and not isinstance(e, threading.BrokenBarrierError):
                raise e
        for e in errs:
            if e is not None:
                raise e
        return res


class _LocalExchange:
    def __init__(self, group, rank):
        self.g, self.rank, self.world = group, rank, group.world

    def _sync(self, t):
        if t.is_cuda:
            torch.cuda.synchronize(t.device)
        self.g.barrier.wait()

    def all_to_all_counts(self, send, el):
        self.g.slots[("cnt", self.rank)] = send
        self._sync(send)
        recv = torch.cat([self.g.slots[("cnt", s)][self.rank * el:(self.rank + 1) * el]
                          for s in range(self.world)]).clone()
        self._sync(send)
        return recv

    def move(self, src, dst, sends, recvs):
        for p, j, off, n in sends:
            self.g.slots[("mv", self.rank, p, j)] = src[off:off + n]
        self._sync(src)
        for p, j, off, n in recvs:
            dst[off:off + n].copy_(self.g.slots[("mv", p, self.rank, j)])
        self._sync(dst)
        for p, j, off, n in sends:
            self.g.slots.pop(("mv", self.rank, p, j), None)

    def all_reduce_sum(self, t):
        self.g.slots[("ar", self.rank)] = t.clone()
        self._sync(t)
        total = self.g.slots[("ar", 0)].clone()
        for s in range(1, self.world):      # fixed order: the same sum on every rank
            total += self.g.slots[("ar", s)]
        self._sync(t)
        t.copy_(total)
        return t


# ------------------------------------------------------------------ the layer
class ExpertParallelMoE:
    """One rank's share of an expert-parallel MoE layer (exact top-k routing).

    forward(x, w_gate, w1, w3, w2): x [T, d] this rank's tokens; w_gate [d, E]
    (replicated); w1, w3 [El, d, f] and w2 [El, f, d] the weights of this
    rank's experts.  backward(dout) returns dx [T, d], dw_gate [d, E] (summed
    over ranks), dw1, dw3, dw2 of the local experts and dlogits [T, E]."""

    def __init__(self, exchange, E, k, ops=None):
        G = exchange.world
        if E % G:
            raise ValueError(f"E = {E} experts do not split evenly over {G} ranks")
        self.ex, self.E, self.k, self.G, self.El = exchange, E, k, G, E // G
        self.ops = ops if ops is not None else CudaOps()

    def _blocks(self, offsets_h, seg_h, recv_rows_h, recv_row_h):
        """(peer, local expert, first row, rows) of every non-empty segment this
        rank sends (from its row space) and receives (into the local rows)."""
        El = self.El
        sends = [(p, j, offsets_h[p * El + j], seg_h[p * El + j])
                 for p in range(self.G) for j in range(El) if seg_h[p * El + j] > 0]
        recvs = [(s, j, recv_row_h[s * El + j], recv_rows_h[s * El + j])
                 for s in range(self.G) for j in range(El) if recv_rows_h[s * El + j] > 0]
        assert all(n % 128 == 0 for *_, n in sends + recvs), "segments are 128-row multiples"
        return sends, recvs

    def forward(self, x, w_gate, w1, w3, w2, logits_override=None):
        ops, E, k, El, G = self.ops, self.E, self.k, self.El, self.G
        T, d = x.shape
        logits, idx, gate = ops.route(x, w_gate, k, logits_override)
        plan = ops.permute(idx, gate, logits, E)
        xg = ops.gather_rows(x, plan, k)
        seg = ops.dispatch_counts(plan["offsets"])
        recv_rows = self.ex.all_to_all_counts(seg, El)
        local_offsets, recv_row = ops.receive_plan(recv_rows.view(G, El))
        # the placement table on the host (one copy per layer): transfers need their sizes
        tab = torch.cat([plan["offsets"].reshape(-1), seg.reshape(-1), recv_rows.reshape(-1),
                         recv_row.reshape(-1), local_offsets.reshape(-1)]).to("cpu").tolist()
        n = [E + 1, E, G * El, G * El, El + 1]
        cut = [sum(n[:i]) for i in range(len(n) + 1)]
        offsets_h, seg_h, recv_rows_h, recv_row_h, loc_h = (tab[cut[i]:cut[i + 1]]
                                                             for i in range(len(n)))
        sends, recvs = self._blocks(offsets_h, seg_h, recv_rows_h, recv_row_h)
        # one rank: the received layout is the row space itself, so the rows stay put
        self.alone = G == 1
        if self.alone:
            rows = max(128, xg.shape[0] // 128 * 128)     # >= offsets[E], a multiple of 128
            xg_loc, gate_loc = xg[:rows], plan["row_gate"][:rows]
        else:
            rows = max(128, loc_h[El])
            xg_loc = torch.empty(rows, d, device=x.device, dtype=x.dtype)
            gate_loc = torch.zeros(rows, device=x.device, dtype=plan["row_gate"].dtype)
            self.ex.move(xg, xg_loc, sends, recvs)
            self.ex.move(plan["row_gate"], gate_loc, sends, recvs)
        H_loc, Y_loc = ops.expert_rows_fwd(xg_loc, w1, w3, w2, local_offsets)
        if self.alone:
            y_perm = Y_loc
        else:
            y_perm = torch.empty_like(xg)
            self.ex.move(Y_loc, y_perm, recvs, sends)      # back to the tokens' ranks
        out = ops.combine(y_perm, plan, T, E, k)
        self._saved = dict(x=x, w_gate=w_gate, w=(w1, w3, w2), logits=logits, idx=idx, gate=gate,
                           plan=plan, xg_loc=xg_loc, gate_loc=gate_loc, H_loc=H_loc,
                           local_offsets=local_offsets, sends=sends, recvs=recvs, rows=rows,
                           router_grad=logits_override is None, cap=xg.shape[0])
        self.routing = dict(logits=logits, idx=idx, gate=gate, plan=plan,
                            local_rows=loc_h[El], local_offsets=local_offsets)
        return out

    def backward(self, dout):
        s, ops, k = self._saved, self.ops, self.k
        T, d = dout.shape
        dog = ops.gather_rows(dout, s["plan"], k)
        if self.alone:
            dog_loc = dog[:s["rows"]]
        else:
            dog_loc = torch.empty(s["rows"], d, device=dout.device, dtype=dout.dtype)
            self.ex.move(dog, dog_loc, s["sends"], s["recvs"])
        w1, w3, w2 = s["w"]
        g = ops.expert_rows_bwd(dog_loc, s["xg_loc"], s["gate_loc"], s["H_loc"], w1, w3, w2,
                                s["local_offsets"])
        if self.alone:
            dx_rows, dS = g["dX_rows"], g["dS"]
        else:
            dx_rows = torch.empty_like(dog)
            dS = torch.zeros(s["cap"], device=dout.device, dtype=g["dS"].dtype)
            self.ex.move(g["dX_rows"], dx_rows, s["recvs"], s["sends"])
            self.ex.move(g["dS"], dS, s["recvs"], s["sends"])
        t = ops.token_bwd(dx_rows, dS, s["x"], s["w_gate"], s["idx"], s["gate"], s["plan"],
                          s["router_grad"])
        dw_gate = self.ex.all_reduce_sum(t["dw_gate"])
        return dict(dx=t["dx"], dw_gate=dw_gate, dlogits=t["dlogits"], dw1=g["dw1"],
                    dw3=g["dw3"], dw2=g["dw2"], dS=dS)
