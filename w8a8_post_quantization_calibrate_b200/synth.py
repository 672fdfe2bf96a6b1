"""Seeded synthetic workloads for the W8A8 smoothed linear layer.

This module only draws random inputs. It holds none of the method's arithmetic
(no maxima, factors, scales or codes), so both the CUDA path and the CPU oracle
can consume its output without sharing any computation.

Outlier model (persistent per-channel outliers, the structure described in
"Why are activations harder to quantize than weights in a transformer?",
"The outlier structure", and built synthetically in the "One outlier" notes,
"Where transformer activations put their outliers"): activations are N(0, 1)
and a seeded set of input channels is multiplied, for every token, by one
per-channel factor. Weights are N(0, sigma) with sigma the standard deviation.

All draws use torch's CPU generator, one seed per workload (1000 + workload
index) and separate sub-streams for activations, weights and outlier choice, so
every run of every test sees the same tensors.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class Outliers:
    """A group of outlier channels: `count` channels (or `frac` of K, rounded),
    each scaled by a factor drawn from `dist` over [lo, hi]."""
    frac: float = 0.0
    count: int | None = None
    dist: str = "fixed"          # "fixed" (lo), "uniform" U[lo,hi], "loguniform" exp(U[ln lo, ln hi])
    lo: float = 1.0
    hi: float = 1.0

    def n_channels(self, K: int) -> int:
        return self.count if self.count is not None else int(round(self.frac * K))


@dataclass(frozen=True)
class Workload:
    name: str
    index: int
    T: int
    K: int
    N: int
    in_dtype: torch.dtype
    out_dtype: torch.dtype
    alpha: float
    w_std: float
    outliers: tuple = field(default_factory=tuple)
    description: str = ""

    @property
    def seed(self) -> int:
        return 1000 + self.index


def _gen(seed: int, stream: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed * 97 + stream)
    return g


# Workload table: shapes, dtypes and outlier recipes of the five benchmark
# configurations (tokens T, input width K, output width N).
WORKLOADS = {
    "tiny": Workload(
        "tiny", 0, T=64, K=1024, N=1024, in_dtype=torch.float32, out_dtype=torch.float32,
        alpha=0.5, w_std=1.0 / 32.0,
        outliers=(Outliers(count=4, dist="fixed", lo=60.0),),
        description="tiny oracle check: X fp32 [64 x 1024], 4 outlier channels x60; "
                    "W fp32 [1024 x 1024] N(0, 1/32); alpha 0.5; fp32 output"),
    "qkv_prefill_7b": Workload(
        "qkv_prefill_7b", 1, T=4096, K=4096, N=12288, in_dtype=torch.bfloat16,
        out_dtype=torch.bfloat16, alpha=0.5, w_std=1.0 / 64.0,
        outliers=(Outliers(frac=0.001, dist="uniform", lo=20.0, hi=80.0),),
        description="7B-like QKV projection prefill: X bf16 [4096 x 4096], 0.1% channels "
                    "x U[20,80]; W bf16 [12288 x 4096] N(0, 1/64); alpha 0.5; bf16 output"),
    "mlp_decode_7b": Workload(
        "mlp_decode_7b", 2, T=16, K=4096, N=11008, in_dtype=torch.bfloat16,
        out_dtype=torch.bfloat16, alpha=0.5, w_std=1.0 / 64.0,
        outliers=(Outliers(frac=0.001, dist="uniform", lo=20.0, hi=80.0),),
        description="7B-like MLP decode: X bf16 [M in {1,8,16} x 4096]; gate/up W "
                    "[11008 x 4096], down W [4096 x 11008], N(0, 1/sqrt(K)); weight streaming"),
    "mlp_prefill_13b_heavy": Workload(
        "mlp_prefill_13b_heavy", 3, T=8192, K=5120, N=13824, in_dtype=torch.bfloat16,
        out_dtype=torch.bfloat16, alpha=0.75, w_std=1.0 / math.sqrt(5120.0),
        outliers=(Outliers(frac=0.30, dist="loguniform", lo=5.0, hi=30.0),
                  Outliers(frac=0.001, dist="fixed", lo=60.0)),
        description="13B-like MLP prefill, heavy outliers: X bf16 [8192 x 5120], 30% "
                    "channels x loguniform[5,30] plus 0.1% x60; W [13824 x 5120]; alpha 0.75"),
    "down_prefill_70b": Workload(
        "down_prefill_70b", 4, T=8192, K=28672, N=8192, in_dtype=torch.bfloat16,
        out_dtype=torch.bfloat16, alpha=0.5, w_std=1.0 / math.sqrt(28672.0),
        outliers=(Outliers(frac=0.0005, dist="uniform", lo=40.0, hi=100.0),),
        description="70B-like down projection prefill: X bf16 [8192 x 28672], 0.05% "
                    "channels x U[40,100]; W [8192 x 28672]; alpha in {0.25,0.5,0.75}; "
                    "calibration over 16 batches of 2048 tokens"),
}

DOWN_70B_ALPHAS = (0.25, 0.5, 0.75)
DOWN_70B_CALIB_BATCHES = 16
DOWN_70B_CALIB_TOKENS = 2048
DECODE_MS = (1, 8, 16)


def outlier_channels(K: int, groups, seed: int):
    """-> (channel index tensor, per-channel factor tensor), disjoint groups."""
    g = _gen(seed, 3)
    perm = torch.randperm(K, generator=g)
    idx, fac = [], []
    start = 0
    for grp in groups:
        n = grp.n_channels(K)
        ch = perm[start:start + n]
        start += n
        u = torch.rand(n, generator=g, dtype=torch.float64)
        if grp.dist == "fixed":
            f = torch.full((n,), grp.lo, dtype=torch.float64)
        elif grp.dist == "uniform":
            f = grp.lo + (grp.hi - grp.lo) * u
        elif grp.dist == "loguniform":
            f = torch.exp(math.log(grp.lo) + (math.log(grp.hi) - math.log(grp.lo)) * u)
        else:
            raise ValueError(grp.dist)
        idx.append(ch)
        fac.append(f)
    if not idx:
        return torch.empty(0, dtype=torch.long), torch.empty(0, dtype=torch.float64)
    return torch.cat(idx), torch.cat(fac)


def activations(T: int, K: int, groups, seed: int, dtype=torch.bfloat16, stream: int = 1):
    """X ~ N(0,1) [T x K] with the outlier channels of `groups` scaled (fp32
    draw, then cast to `dtype`)."""
    x = torch.randn(T, K, generator=_gen(seed, stream), dtype=torch.float32)
    ch, f = outlier_channels(K, groups, seed)
    if ch.numel():
        x[:, ch] *= f.to(torch.float32)
    return x.to(dtype)


def weights(N: int, K: int, std: float, seed: int, dtype=torch.bfloat16, stream: int = 2):
    w = torch.randn(N, K, generator=_gen(seed, stream), dtype=torch.float32)
    w *= std
    return w.to(dtype)


def make(name: str, T: int | None = None, N: int | None = None, K: int | None = None):
    """Draw (X, W) for a named workload, optionally with overridden sizes (the
    override keeps the workload's recipe and seed)."""
    wl = WORKLOADS[name]
    T = wl.T if T is None else T
    K = wl.K if K is None else K
    N = wl.N if N is None else N
    x = activations(T, K, wl.outliers, wl.seed, wl.in_dtype)
    w = weights(N, K, wl.w_std, wl.seed, wl.in_dtype)
    return x, w


def make_decode(M: int, which: str):
    """7B-like MLP decode: `which` in {"gate", "up", "down"}; gate/up are
    [11008 x 4096], down is [4096 x 11008]; sigma = 1/sqrt(K)."""
    wl = WORKLOADS["mlp_decode_7b"]
    if which in ("gate", "up"):
        N, K = 11008, 4096
    elif which == "down":
        N, K = 4096, 11008
    else:
        raise ValueError(which)
    stream_w = {"gate": 2, "up": 4, "down": 5}[which]
    x = activations(M, K, wl.outliers, wl.seed + 100 * (K != 4096), wl.in_dtype)
    w = weights(N, K, 1.0 / math.sqrt(K), wl.seed, wl.in_dtype, stream=stream_w)
    return x, w


def calibration_batches(name: str = "down_prefill_70b", n_batches: int = DOWN_70B_CALIB_BATCHES,
                        tokens: int = DOWN_70B_CALIB_TOKENS, K: int | None = None):
    """Calibration batches from the same activation model (same outlier
    channels and factors, fresh N(0,1) draws per batch)."""
    wl = WORKLOADS[name]
    K = wl.K if K is None else K
    for b in range(n_batches):
        yield activations(tokens, K, wl.outliers, wl.seed, wl.in_dtype, stream=10 + b)


def outlier_experiment_inputs():
    """The seeded synthetic test of the inferenceinterviews page ("A strong
    answer"): X ~ N(0,1) [512 x 4096] with 6 channels x60, W ~ N(0,1)*0.02
    [1024 x 4096], drawn with numpy's default_rng(0) in that order, fp64."""
    rng = np.random.default_rng(0)
    X = rng.normal(size=(512, 4096))
    ch = rng.choice(4096, 6, replace=False)
    X[:, ch] *= 60
    W = rng.normal(size=(1024, 4096)) * 0.02
    return X, W


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw uint16 bit patterns of a CPU bf16 tensor (for the oracle)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def host_array(t: torch.Tensor) -> np.ndarray:
    """CPU tensor -> numpy array the oracle accepts (fp32, or bf16 bits)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return bf16_bits(t)
    return t.numpy()
