"""The N > 1 host path of bench.py on CPU: two ranks on the gloo backend
(127.0.0.1) take the slowest replica's time (max over ranks) and report the
whole-job throughput; the reference arm runs on rank 0 only."""
import json
import os
import socket
import subprocess
import sys
import textwrap

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

WORKER = textwrap.dedent("""
    import datetime, json, os, sys
    sys.path.insert(0, {root!r})
    import torch.distributed as dist
    import bench
    rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        total = bench.max_over_ranks(100.0 + 50.0 * rank, world)     # rank 1 is slower
        e2e = bench.max_over_ranks(7.0 * (world - rank), world)       # rank 0 is slower here
        rate = bench.job_tokens_per_s(world, 1000, 10, total)
        dist.barrier()
        print(json.dumps({{"rank": rank, "total": total, "e2e": e2e, "rate": rate}}), flush=True)
    finally:
        dist.destroy_process_group()
""")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_take_the_slowest_replica(tmp_path):
    script = tmp_path / "worker.py"
    script.write_text(WORKER.format(root=ROOT))
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, str(script)], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        try:
            out, err = p.communicate(timeout=180)
        except subprocess.TimeoutExpired:
            for q in procs:
                q.kill()
            raise
        assert p.returncode == 0, err
        outs.append(json.loads(out.strip().splitlines()[-1]))
    for o in outs:
        assert o["total"] == 150.0            # the slower rank's time, on every rank
        assert o["e2e"] == 14.0
        assert o["rate"] == pytest.approx(2 * 1000 * 10 / 0.150)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(12.5, 1) == 12.5
    assert bench.job_tokens_per_s(1, 16384, 200, 500.0) == pytest.approx(16384 * 200 / 0.5)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    # any rank but 0 exits at once, without work and without output
    assert bench.run_reference(None, None, rank=1, world=2) == 0
    assert capsys.readouterr().out == ""
