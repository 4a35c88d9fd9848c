"""Expert parallelism (mixture_experts_layer_59_b200.ep) on CPU ranks.

The exchange and placement logic of ExpertParallelMoE runs with the oracle's
compute ops (float64, no staging): G ranks each own E/G experts and T
tokens; their outputs, dx, dlogits and local expert gradients must equal the
oracle's one-device layer on all G*T tokens, and dW_gate (summed over ranks)
its router gradient.  Two real gloo ranks (separate processes, 127.0.0.1)
and G = 1, 2, 4 ranks as threads of one process."""
import json
import os
import socket
import subprocess
import sys
import textwrap

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.join(ROOT, "tests"))

import ep_oracle_ops as EO  # noqa: E402
from mixture_experts_layer_59_b200.ep import LocalGroup  # noqa: E402

# tokens per rank, d, f, E, k: small enough for the pure-numpy oracle
SHAPE = dict(T=96, d=64, f=32, E=8, k=2)


def _check(results, G, T, d, f, E, k, seed=0):
    x, dout, wg, w1, w3, w2 = EO.make_problem(G, T, d, f, E, k, seed)
    fwd, bwd = EO.reference(x, dout, wg, w1, w3, w2, k)
    El = E // G
    tol = dict(rtol=1e-9, atol=1e-11)
    for r, res in enumerate(results):
        sl, el = slice(r * T, (r + 1) * T), slice(r * El, (r + 1) * El)
        np.testing.assert_allclose(res["out"], fwd["out"][sl], **tol, err_msg=f"out rank {r}")
        np.testing.assert_allclose(res["dx"], bwd["dx"][sl], **tol, err_msg=f"dx rank {r}")
        np.testing.assert_allclose(res["dlogits"], bwd["dlogits"][sl], **tol)
        np.testing.assert_allclose(res["dw_gate"], bwd["dw_gate"], **tol)
        for n in ("dw1", "dw3", "dw2"):
            np.testing.assert_allclose(res[n], bwd[n][el], **tol, err_msg=f"{n} rank {r}")
    # every routed row reached exactly one expert's rank: the local row counts
    # add up to the global plan's padded segments regrouped by rank
    counts = np.bincount(fwd["idx"].ravel(), minlength=E)
    per_rank_tok = [np.bincount(fwd["idx"][r * T:(r + 1) * T].ravel(), minlength=E)
                    for r in range(G)]
    pad = lambda n: (n + 127) // 128 * 128
    for g in range(G):
        want = sum(pad(per_rank_tok[s][e]) for s in range(G) for e in range(g * El, (g + 1) * El))
        assert results[g]["local_rows"] == want
    assert sum(c.sum() for c in per_rank_tok) == counts.sum() == G * T * k


@pytest.mark.parametrize("G", [1, 2, 4])
def test_ep_threads_match_the_one_device_layer(G):
    s = SHAPE
    grp = LocalGroup(G, timeout=60)
    res = grp.run(lambda r, ex: EO.run_rank(r, ex, G, s["T"], s["d"], s["f"], s["E"], s["k"], 3))
    _check(res, G, s["T"], s["d"], s["f"], s["E"], s["k"], 3)


def test_ep_rejects_uneven_expert_split():
    from mixture_experts_layer_59_b200.ep import ExpertParallelMoE
    grp = LocalGroup(3)
    with pytest.raises(ValueError):
        ExpertParallelMoE(grp.member(0), 8, 2, ops=EO.OracleOps())


def test_ep_rank_failure_breaks_the_others_out():
    """A rank that raises mid-step aborts the group's barrier: the other ranks
    leave their next exchange with an error instead of waiting forever."""
    grp = LocalGroup(2, timeout=30)

    def fn(r, ex):
        if r == 1:
            raise RuntimeError("rank 1 failed before its first exchange")
        return EO.run_rank(r, ex, 2, 32, 64, 32, 8, 2)

    with pytest.raises(RuntimeError, match="rank 1 failed"):
        grp.run(fn)


WORKER = textwrap.dedent("""
    import datetime, json, os, sys
    sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
    import numpy as np
    import torch.distributed as dist
    import ep_oracle_ops as EO
    from mixture_experts_layer_59_b200.ep import TorchDistExchange
    rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        res = EO.run_rank(rank, TorchDistExchange(), world, {T}, {d}, {f}, {E}, {k}, 5)
        np.savez({out!r} + f"_{{rank}}.npz", **res)
        dist.barrier()
        print(json.dumps({{"rank": rank, "ok": True}}), flush=True)
    finally:
        dist.destroy_process_group()
""")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_ep_two_gloo_ranks_match_the_one_device_layer(tmp_path):
    s = SHAPE
    script = tmp_path / "worker.py"
    out = str(tmp_path / "res")
    script.write_text(WORKER.format(root=ROOT, tests=os.path.join(ROOT, "tests"), out=out, **s))
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, str(script)], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = [p.communicate(timeout=240) for p in procs]
    for p, (o, e) in zip(procs, outs):
        assert p.returncode == 0, e[-2000:]
        assert json.loads(o.strip().splitlines()[-1])["ok"]
    res = [dict(np.load(f"{out}_{r}.npz")) for r in range(2)]
    for r in res:
        r["local_rows"] = int(r["local_rows"])
    _check(res, 2, s["T"], s["d"], s["f"], s["E"], s["k"], 5)


def test_ep_rank_with_no_rows_gets_zero_expert_gradients():
    """Routing that sends every token to the first rank's experts: the other
    rank receives no rows, its grouped GEMMs see empty segments, and its
    expert gradients come back zero; the layer still matches the oracle."""
    import torch
    from mixture_experts_layer_59_b200.ep import ExpertParallelMoE
    G, T, d, f, E, k = 2, 64, 64, 32, 4, 2
    x, dout, wg, w1, w3, w2 = EO.make_problem(G, T, d, f, E, k, 9)
    lo = np.full((G * T, E), -5.0)
    lo[:, 0], lo[:, 1] = 1.0, 0.5               # experts 0 and 1 live on rank 0
    lo += 1e-3 * np.random.default_rng(9).standard_normal(lo.shape)
    El = E // G
    t = torch.from_numpy

    def fn(r, ex):
        sl, el = slice(r * T, (r + 1) * T), slice(r * El, (r + 1) * El)
        layer = ExpertParallelMoE(ex, E, k, ops=EO.OracleOps())
        out = layer.forward(t(x[sl]), t(wg), t(w1[el]), t(w3[el]), t(w2[el]),
                            logits_override=t(lo[sl]))
        g = layer.backward(t(dout[sl]))
        return dict(out=out.numpy(), dx=g["dx"].numpy(), dw1=g["dw1"].numpy(),
                    dw2=g["dw2"].numpy(), local_rows=layer.routing["local_rows"])

    res = LocalGroup(G, timeout=60).run(fn)
    from oracle import moe_oracle as O
    fwd = O.layer_fwd(x, wg, w1, w3, w2, k, logits_override=lo, staged=False)
    bwd = O.layer_bwd(dout, x, wg, w1, w3, w2, fwd, staged=False, router_grad_on=False)
    assert res[1]["local_rows"] == 0
    assert not res[1]["dw1"].any() and not res[1]["dw2"].any()
    for r in range(G):
        sl, el = slice(r * T, (r + 1) * T), slice(r * El, (r + 1) * El)
        np.testing.assert_allclose(res[r]["out"], fwd["out"][sl], rtol=1e-9, atol=1e-11)
        np.testing.assert_allclose(res[r]["dx"], bwd["dx"][sl], rtol=1e-9, atol=1e-11)
        np.testing.assert_allclose(res[r]["dw1"], bwd["dw1"][el], rtol=1e-9, atol=1e-11)
