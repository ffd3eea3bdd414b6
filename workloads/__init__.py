"""Seeded synthetic inputs for the DeepSeekMoE FP8 layer.

This module only draws random numbers. It holds none of the layer's
arithmetic (no routing, no quantisation, no GEMM): both the CUDA path and the
CPU oracle receive the tensors made here and each computes on its own.

Five workloads are defined, with the shapes of the DeepSeek-V3 MoE layer
("DeepSeek-V3 Teknik Raporu", Temel fikirler: 1 shared + 256 routed experts,
8 active) and scaled-down variants of it:

    name     T      d     N_r  K_r  I     activations
    tiny     64     256   8    2    128   N(0,1)
    mid      4096   2048  64   6    1024  N(0,1)
    prefill  8192   7168  256  8    2048  N(0,1), 0.1% of channels x50
    decode   128    7168  256  8    2048  N(0,1)
    skew     16384  7168  256  8    2048  Student-t (df=3) + common direction

Weights are N(0, 0.02) (std 0.02) in FP32 before quantisation; router
centroids are N(0, 1/d) (variance 1/d, so logits are ~N(0,1)); all other
recipe details are in the generator functions below.

Random streams come from ``torch.Generator`` on the requested device. CPU and
CUDA generators give different numbers for the same seed, so a test must hand
the *same* tensors to both sides (copying to the host what the oracle needs).
"""
from __future__ import annotations

import json
import math
import os
from dataclasses import dataclass, replace

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))


@dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int          # tokens in the batch
    d: int          # hidden size
    N_r: int        # routed experts
    K_r: int        # experts selected per token
    I: int          # expert intermediate size (SwiGLU)
    seed: int
    act: str = "normal"        # normal | normal_outliers | student_t
    bias: str = "zero"         # zero | uniform001 | normal001
    N_s: int = 1               # shared experts (always 1 here)

    @property
    def P(self) -> int:
        """Rows after permutation: one per (token, selected expert)."""
        return self.T * self.K_r

    def with_tokens(self, T: int) -> "MoEConfig":
        return replace(self, T=T)


CONFIGS = {
    "tiny": MoEConfig("tiny", T=64, d=256, N_r=8, K_r=2, I=128, seed=0),
    "mid": MoEConfig("mid", T=4096, d=2048, N_r=64, K_r=6, I=1024, seed=1,
                     bias="uniform001"),
    "prefill": MoEConfig("prefill", T=8192, d=7168, N_r=256, K_r=8, I=2048,
                         seed=2, act="normal_outliers", bias="normal001"),
    "decode": MoEConfig("decode", T=128, d=7168, N_r=256, K_r=8, I=2048,
                        seed=3),
    "skew": MoEConfig("skew", T=16384, d=7168, N_r=256, K_r=8, I=2048, seed=4,
                      act="student_t"),
}

WEIGHT_STD = 0.02
OUTLIER_FRACTION = 0.001
OUTLIER_GAIN = 50.0
SKEW_HOT_FRACTION = 0.10


def _gen(device, *key: int) -> torch.Generator:
    """A generator seeded from a tuple of small integers."""
    s = 0x9E3779B1
    for k in key:
        s = (s * 1_000_003 + int(k) + 1) % (2**61 - 1)
    g = torch.Generator(device=device)
    g.manual_seed(s)
    return g


# stream ids inside one config
_S_ACT, _S_OUTLIER, _S_CENT, _S_BIAS, _S_HOT, _S_DIR, _S_CHI = range(7)
_S_WEIGHT = 100


def _skew_params() -> dict:
    """Hot-set shift for the skew workload, calibrated by a committed script
    (tests/golden/make_skew_calibration.py) that runs only the CPU oracle."""
    path = os.path.join(_HERE, "..", "tests", "golden", "skew_calibration.json")
    with open(path) as f:
        return json.load(f)


def _direction(cfg: MoEConfig, device) -> torch.Tensor:
    v = torch.randn(cfg.d, generator=_gen(device, cfg.seed, _S_DIR),
                    device=device, dtype=torch.float32)
    return v / v.norm()


def hot_experts(cfg: MoEConfig, device="cpu") -> torch.Tensor:
    """Indices of the over-popular experts of the skew workload (10%)."""
    n_hot = max(1, round(SKEW_HOT_FRACTION * cfg.N_r))
    perm = torch.randperm(cfg.N_r, generator=_gen("cpu", cfg.seed, _S_HOT))
    return perm[:n_hot].sort().values.to(device)


def activations(cfg: MoEConfig, device="cpu", skew: dict | None = None
                ) -> torch.Tensor:
    """u: [T, d] bf16."""
    g = _gen(device, cfg.seed, _S_ACT)
    x = torch.randn(cfg.T, cfg.d, generator=g, device=device,
                    dtype=torch.float32)
    if cfg.act == "normal_outliers":
        n_out = max(1, round(OUTLIER_FRACTION * cfg.d))
        ch = torch.randperm(cfg.d, generator=_gen("cpu", cfg.seed, _S_OUTLIER))
        x[:, ch[:n_out].to(device)] *= OUTLIER_GAIN
    elif cfg.act == "student_t":
        # Student-t with 3 degrees of freedom: z / sqrt(chi2_3 / 3)
        gc = _gen(device, cfg.seed, _S_CHI)
        chi = torch.zeros_like(x)
        for _ in range(3):
            chi += torch.randn(x.shape, generator=gc, device=device,
                               dtype=torch.float32) ** 2
        x = x / torch.sqrt(chi / 3.0)
        p = skew if skew is not None else _skew_params()
        x += float(p["m"]) * _direction(cfg, device)[None, :]
    elif cfg.act != "normal":
        raise ValueError(cfg.act)
    return x.to(torch.bfloat16)


def centroids(cfg: MoEConfig, device="cpu", skew: dict | None = None
              ) -> torch.Tensor:
    """e: [N_r, d] bf16, N(0, 1/d)."""
    g = _gen(device, cfg.seed, _S_CENT)
    e = torch.randn(cfg.N_r, cfg.d, generator=g, device=device,
                    dtype=torch.float32) / math.sqrt(cfg.d)
    if cfg.act == "student_t":
        p = skew if skew is not None else _skew_params()
        hot = hot_experts(cfg, device)
        e[hot] += float(p["beta"]) * _direction(cfg, device)[None, :]
    return e.to(torch.bfloat16)


def bias(cfg: MoEConfig, device="cpu") -> torch.Tensor:
    """b: [N_r] fp32 routing bias at step 0."""
    g = _gen(device, cfg.seed, _S_BIAS)
    if cfg.bias == "zero":
        return torch.zeros(cfg.N_r, device=device, dtype=torch.float32)
    if cfg.bias == "uniform001":
        return (torch.rand(cfg.N_r, generator=g, device=device,
                           dtype=torch.float32) * 0.02 - 0.01)
    if cfg.bias == "normal001":
        return torch.randn(cfg.N_r, generator=g, device=device,
                           dtype=torch.float32) * 0.01
    raise ValueError(cfg.bias)


def expert_weights(cfg: MoEConfig, slot: int, device="cpu"):
    """FP32 weights of one expert before quantisation.

    slot in [0, N_r) is a routed expert, slot == N_r the shared expert.
    Returns (W_gate [I, d], W_up [I, d], W_down [d, I]).
    """
    if not 0 <= slot <= cfg.N_r:
        raise ValueError(slot)
    out = []
    for k, shape in enumerate([(cfg.I, cfg.d), (cfg.I, cfg.d), (cfg.d, cfg.I)]):
        g = _gen(device, cfg.seed, _S_WEIGHT, slot, k)
        out.append(torch.randn(shape, generator=g, device=device,
                               dtype=torch.float32) * WEIGHT_STD)
    return tuple(out)


def scores(T: int, N_r: int, seed: int, device="cpu", ties: bool = False
           ) -> torch.Tensor:
    """Stand-alone FP32 affinity matrix in (0, 1) for top-K tests.

    With ties=True the values are drawn from a 16-level grid so that equal
    keys are common and the lower-index tie rule is exercised.
    """
    g = _gen(device, seed, 7777)
    if ties:
        lv = torch.randint(1, 16, (T, N_r), generator=g, device=device)
        return lv.to(torch.float32) / 16.0
    return torch.rand(T, N_r, generator=g, device=device,
                      dtype=torch.float32) * 0.98 + 0.01


def topk_indices(T: int, N_r: int, K_r: int, seed: int, device="cpu",
                 pattern: str = "uniform") -> torch.Tensor:
    """Synthetic expert choices [T, K_r] int32 (distinct per row) for
    permutation tests. pattern: uniform | one_hot_expert | first_k."""
    g = _gen("cpu", seed, 8888)
    if pattern == "uniform":
        idx = torch.argsort(torch.rand(T, N_r, generator=g), dim=1)[:, :K_r]
    elif pattern == "first_k":
        idx = torch.arange(K_r).repeat(T, 1)
    elif pattern == "one_hot_expert":
        # every token picks expert 0 plus K_r-1 others
        rest = torch.argsort(torch.rand(T, N_r - 1, generator=g), dim=1)
        idx = torch.cat([torch.zeros(T, 1, dtype=torch.long),
                         rest[:, :K_r - 1] + 1], dim=1)
    else:
        raise ValueError(pattern)
    return idx.to(torch.int32).to(device)
