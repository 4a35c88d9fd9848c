"""CPU checks of the seeded input generator (deterministic; one stream per
tensor, so one tensor's shape never changes another's values) and of the
reference arm's JSON line, which the driver parses."""
import json
import os
import subprocess
import sys

import torch

from mixture_experts_layer_59_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_inputs_are_deterministic_and_streams_independent():
    cfg = synth.MoEConfig("t", 64, 128, 64, 8, 2, std=0.05, routing="zipf")
    a = synth.make_inputs(cfg, seed=5)
    b = synth.make_inputs(cfg, seed=5)
    for n, t in a.items():
        if t is not None:
            assert torch.equal(t, b[n]), n
    # a different d_ff changes the expert weights' shapes only
    c = synth.make_inputs(cfg.with_(f=96), seed=5)
    for n in ("x", "w_gate", "dout", "logit_bias"):
        assert torch.equal(a[n], c[n]), n
    # a different seed changes every drawn tensor
    d = synth.make_inputs(cfg, seed=6)
    for n in ("x", "w_gate", "w1", "w3", "w2", "dout"):
        assert not torch.equal(a[n], d[n]), n
    assert a["x"].dtype == torch.bfloat16 and a["w1"].shape == (8, 128, 64)


def test_noise_is_seeded():
    assert torch.equal(synth.logit_noise(16, 8, 0.5, seed=2), synth.logit_noise(16, 8, 0.5, seed=2))
    assert not torch.equal(synth.logit_noise(16, 8, 0.5, seed=2), synth.logit_noise(16, 8, 0.5, seed=3))


def test_reference_arm_prints_one_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny_fp32", "--steps", "1", "--warmup", "1",
                        "--ref-sample", "32"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["unit"] == "tokens/s" and j["value"] > 0
    assert j["steps"] == 1 and j["warmup"] == 1 and j["higher_is_better"] is True
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["value"] == j["value"]
    assert j["e2e"] == {"value": j["value"], "unit": "tokens/s",
                        "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert j["config"]["workload"] == "tiny_fp32"
