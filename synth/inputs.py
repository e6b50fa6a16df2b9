"""Seeded synthetic input recipes (no method arithmetic here).

Workload shapes follow the pages:
  * activations: per-token rows of N(0,1) with a handful of outlier channels
    scaled by a large factor ("Kimi 2.7 MoE, 4-bit storage to INT8" §3.3 on
    activation outliers; "Inference Quantization ch.1" §5 outlier example);
  * weights: N(0, 0.02) fp32, optionally with a Bernoulli(p) mask of entries
    multiplied by a factor (rare large weights);
  * router logits: N(0,1), optionally skewed by log of a Zipf(alpha) law over a
    random rank permutation of the experts.

Everything is generated on the CPU with torch.Generator unless a CUDA device
is given (used only for the very large expert stacks, where the bytes are
generated once on the device and copied back for whatever the oracle checks).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass
class LinearInputs:
    X: torch.Tensor          # bf16 [M, K]
    W: torch.Tensor          # fp32 [K, N]
    outlier_channels: torch.Tensor  # int64 [n_outliers]


@dataclasses.dataclass
class MoEInputs:
    X: torch.Tensor          # bf16 [T, H]
    logits: torch.Tensor     # fp32 [T, E]
    outlier_channels: torch.Tensor


# Named workloads (the shapes and distributions of the pages' workloads).
CONFIGS = {
    "linear_small": dict(M=16, K=512, N=512, group=128, symmetric=True,
                         n_outliers=0, outlier_scale=1.0, seed=0),
    "linear_decode": dict(M=32, K=4096, N=14336, group=128, symmetric=True,
                          n_outliers=8, outlier_scale=50.0, seed=0),
    "linear_prefill": dict(M=8192, K=4096, N=14336, group=128, symmetric=True,
                           n_outliers=8, outlier_scale=50.0, seed=0),
    "moe_sym": dict(T=4096, H=2048, E=64, topk=6, I=1408, group=128,
                    symmetric=True, zipf=None, w_outlier_p=0.0, seed=0),
    "moe_asym_decode": dict(T=64, H=7168, E=256, topk=8, I=2048, group=64,
                            symmetric=False, zipf=1.1, w_outlier_p=0.001, seed=0),
    "moe_asym_prefill": dict(T=8192, H=7168, E=256, topk=8, I=2048, group=64,
                             symmetric=False, zipf=1.1, w_outlier_p=0.001, seed=0),
    # the asymmetric prefill layer scaled down for counter captures: the same
    # shapes per expert and the same mean rows per expert (T * topk / E = 256)
    # with 1/8 of the experts and tokens (about 0.7 GB of packed weights)
    "moe_asym_prefill_e32": dict(T=1024, H=7168, E=32, topk=8, I=2048, group=64,
                                 symmetric=False, zipf=1.1, w_outlier_p=0.001, seed=0),
}


def _gen(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _activations(g: torch.Generator, rows: int, K: int, n_outliers: int,
                 outlier_scale: float, device="cpu"):
    X = torch.randn(rows, K, generator=g, dtype=torch.float32, device=device)
    if n_outliers > 0:
        ch = torch.randperm(K, generator=g, device=device)[:n_outliers]
        X[:, ch] *= outlier_scale
    else:
        ch = torch.empty(0, dtype=torch.int64, device=device)
    return X.to(torch.bfloat16), ch


def _weight(g: torch.Generator, K: int, N: int, std: float, outlier_p: float,
            outlier_scale: float, device="cpu"):
    W = torch.randn(K, N, generator=g, dtype=torch.float32, device=device) * std
    if outlier_p > 0.0:
        mask = torch.rand(K, N, generator=g, device=device) < outlier_p
        W = torch.where(mask, W * outlier_scale, W)
    return W


def gen_linear(M: int, K: int, N: int, seed: int = 0, n_outliers: int = 8,
               outlier_scale: float = 50.0, w_std: float = 0.02,
               device="cpu") -> LinearInputs:
    """X bf16 [M,K] ~ N(0,1) with `n_outliers` channels x `outlier_scale`;
    W fp32 [K,N] ~ N(0, w_std)."""
    g = _gen(seed, device)
    X, ch = _activations(g, M, K, n_outliers, outlier_scale, device)
    W = _weight(g, K, N, w_std, 0.0, 1.0, device)
    return LinearInputs(X=X, W=W, outlier_channels=ch)


def zipf_logits(g: torch.Generator, T: int, E: int, alpha: Optional[float],
                device="cpu") -> torch.Tensor:
    """N(0,1) logits, plus log(r_e^-alpha / H_E(alpha)) for a random rank
    permutation r of 1..E when alpha is given."""
    L = torch.randn(T, E, generator=g, dtype=torch.float32, device=device)
    if alpha is not None:
        r = torch.randperm(E, generator=g, device=device).to(torch.float64) + 1.0
        h = sum(float(i) ** (-alpha) for i in range(1, E + 1))
        bias = torch.log(r.pow(-alpha) / h).to(torch.float32)
        L = L + bias[None, :]
    return L


def gen_moe_activations(T: int, H: int, E: int, seed: int = 0,
                        zipf: Optional[float] = None, n_outliers: int = 8,
                        outlier_scale: float = 50.0, device="cpu") -> MoEInputs:
    """Token activations and router logits for one MoE layer call."""
    g = _gen(seed, device)
    X, ch = _activations(g, T, H, n_outliers, outlier_scale, device)
    logits = zipf_logits(g, T, E, zipf, device)
    return MoEInputs(X=X, logits=logits, outlier_channels=ch)


def gen_expert_weight(seed: int, expert: int, which: int, K: int, N: int,
                      outlier_p: float = 0.0, outlier_scale: float = 20.0,
                      w_std: float = 0.02, device="cpu") -> torch.Tensor:
    """fp32 [K,N] weight of one expert matrix (which=0: gate_up, 1: down),
    from its own generator so any single expert can be regenerated alone."""
    sub = (int(seed) * 1_000_003 + int(expert) * 2 + int(which) + 17) % (2 ** 62)
    g = _gen(sub, device)
    return _weight(g, K, N, w_std, outlier_p, outlier_scale, device)


def harmonic(E: int, alpha: float) -> float:
    return math.fsum(float(i) ** (-alpha) for i in range(1, E + 1))
