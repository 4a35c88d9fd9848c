"""Seeded synthetic inputs for the token-choice MoE layer.

This module only draws random tensors with the shapes, scales and routing
patterns of the workloads; it holds none of the layer's arithmetic, so both
the CUDA path and the CPU oracle may take their inputs from it.

Workloads (all seeded, no datasets, no trained weights):

* ``tiny_fp32``  T=256,   d=128,  f=256,  E=8,   k=2, fp32, x~N(0,1),
  W_gate,W1,W3~N(0,1/d), W2~N(0,1/f), dO~N(0,1).
* ``coarse``     T=16384, d=2048, f=1024, E=8,   k=4, bf16, weights N(0,0.02^2).
* ``pool``       T=16384, d=2048, f=1024, E=128, k=4, bf16.
* ``fine``       T=32768, d=1536, f=256,  E=64,  k=8, bf16.
* ``sparse``     T=8192,  d=7168, f=2048, E=256, k=8, bf16, Zipf(1.1) expert bias.

Routing variants: ``learned`` (logits = x.W_gate), ``uniform`` (logits drawn
i.i.d. U(0,1), the random-routing system benchmark), ``gauss`` (i.i.d. N(0,1)
logits) and ``zipf`` (learned logits plus a per-expert bias -s*ln(rank_e),
rank_e a seeded permutation of 1..E, which makes expert loads Zipf-skewed)
and ``balanced`` (token t scores experts (t*k + j) mod E, j < k, above all
others, so every expert receives exactly T*k/E rows when E divides T*k: a
load-balanced router, used to time the grouped GEMMs at a fixed row count
per expert).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int
    d: int
    f: int
    E: int
    k: int
    dtype: str = "bf16"          # "bf16" or "f32"
    init: str = "fixed"          # "fixed": N(0, std^2) everywhere; "fan_in": N(0, 1/fan_in)
    std: float = 0.02
    routing: str = "learned"     # learned | uniform | gauss | zipf | balanced
    zipf_s: float = 1.1

    def with_(self, **kw) -> "MoEConfig":
        return replace(self, **kw)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


CONFIGS = {
    "tiny_fp32": MoEConfig("tiny_fp32", 256, 128, 256, 8, 2, dtype="f32", init="fan_in"),
    "coarse": MoEConfig("coarse", 16384, 2048, 1024, 8, 4),
    "pool": MoEConfig("pool", 16384, 2048, 1024, 128, 4, routing="uniform"),
    "fine": MoEConfig("fine", 32768, 1536, 256, 64, 8),
    "sparse": MoEConfig("sparse", 8192, 7168, 2048, 256, 8, routing="zipf"),
}

# One stream id per drawn tensor, so that changing one tensor's shape never
# changes another tensor's values.
_STREAMS = {"x": 1, "w_gate": 2, "w1": 3, "w3": 4, "w2": 5, "dout": 6,
            "logits": 7, "zipf_rank": 8, "noise": 9}


def _gen(seed: int, stream: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + _STREAMS[stream] * 7919) & 0x7FFF_FFFF_FFFF)
    return g


def _normal(shape, std, dtype, seed, stream, device):
    g = _gen(seed, stream, device)
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def make_inputs(cfg: MoEConfig, seed: int = 0, device="cpu") -> dict:
    """Draw every input of one forward+backward pass of the layer.

    Returns x[T,d], w_gate[d,E], w1[E,d,f], w3[E,d,f], w2[E,f,d], dout[T,d]
    in the config's dtype, plus ``logits_override`` ([T,E] fp32 or None) and
    ``logit_bias`` ([E] fp32 or None) that encode the routing variant.
    """
    dt = cfg.torch_dtype
    T, d, f, E = cfg.T, cfg.d, cfg.f, cfg.E
    if cfg.init == "fan_in":
        s_in, s_out = 1.0 / math.sqrt(d), 1.0 / math.sqrt(f)
    else:
        s_in = s_out = cfg.std
    out = {
        "x": _normal((T, d), 1.0, dt, seed, "x", device),
        "w_gate": _normal((d, E), s_in, dt, seed, "w_gate", device),
        "w1": _normal((E, d, f), s_in, dt, seed, "w1", device),
        "w3": _normal((E, d, f), s_in, dt, seed, "w3", device),
        "w2": _normal((E, f, d), s_out, dt, seed, "w2", device),
        "dout": _normal((T, d), 1.0, dt, seed, "dout", device),
        "logits_override": None,
        "logit_bias": None,
    }
    if cfg.routing == "uniform":
        g = _gen(seed, "logits", device)
        out["logits_override"] = torch.rand((T, E), generator=g, device=device, dtype=torch.float32)
    elif cfg.routing == "gauss":
        out["logits_override"] = _normal((T, E), 1.0, torch.float32, seed, "logits", device)
    elif cfg.routing == "zipf":
        g = _gen(seed, "zipf_rank", "cpu")
        rank = torch.randperm(E, generator=g).to(torch.float64) + 1.0
        out["logit_bias"] = (-cfg.zipf_s * torch.log(rank)).to(torch.float32).to(device)
    elif cfg.routing == "balanced":
        t = torch.arange(T, device=device)
        lo = torch.zeros((T, E), device=device, dtype=torch.float32)
        for j in range(cfg.k):
            lo[t, (t * cfg.k + j) % E] = 2.0 - 1e-3 * j
        out["logits_override"] = lo
    elif cfg.routing != "learned":
        raise ValueError(f"unknown routing variant {cfg.routing!r}")
    return out


def quantized_logits(T: int, E: int, levels: int, seed: int = 0) -> torch.Tensor:
    """fp32 logits drawn from a small set of values, so that many exact ties
    occur; used to exercise the lowest-expert-id tie rule."""
    g = _gen(seed, "logits", "cpu")
    return torch.randint(0, levels, (T, E), generator=g).to(torch.float32) * 0.25


def logit_noise(T: int, E: int, std: float, seed: int = 0, device="cpu") -> torch.Tensor:
    """Gaussian routing noise eps ~ N(0, std^2) [T,E] fp32 for noisy top-k
    gating: the random numbers the method draws, handed to both sides."""
    return _normal((T, E), std, torch.float32, seed, "noise", device)
