"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle.

This module holds none of the MLP's arithmetic: it only draws random numbers
(numpy PCG64) and rounds them to BF16 storage with torch's CPU cast, so that
the CUDA path and the CPU oracle receive bit-identical operands.  BF16
tensors are returned as ``uint16`` bit patterns.

Workloads follow the 768-dim GPT-2-small / nanochat MLP shapes the pages
train (d=768, h=4d; 9-layer stack; about 131072 tokens per step).  The
``grid`` distributions draw small integers times powers of two, so that every
partial sum of the up-projection is exact in fp32 whatever the summation
order; they make post, the FP8 codes and the amax comparable bit for bit.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch


def to_bf16_bits(a) -> np.ndarray:
    """fp32 -> BF16 bit patterns (torch CPU cast, round-to-nearest-even)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


@dataclass(frozen=True)
class Workload:
    name: str
    M: int
    d: int
    h: int
    steps: int = 1
    layers: int = 1
    margin: float = 2.0
    x_dist: str = "normal"          # normal | student_t3 | grid
    w_dist: str = "normal"          # normal | grid
    perturb_var: float = 0.0        # variance of the per-step weight perturbation
    spike_steps: tuple = field(default_factory=tuple)
    spike_factor: float = 1.0       # x multiplier at spike steps (post scales by its square)
    backward: bool = True
    description: str = ""


WORKLOADS = {
    "tiny": Workload(
        "tiny", M=256, d=64, h=256, steps=3, perturb_var=1e-3,
        description="M=256 d=64 h=256, x~N(0,1), W1~N(0,1/d), W2~N(0,1/h), "
                    "dOut~N(0,1), 3 delayed-scaling steps, margin 2, "
                    "W1/W2 += N(0,1e-3) per step, seed 0"),
    "fwd16k": Workload(
        "fwd16k", M=16384, d=768, h=3072, backward=False,
        description="GPT-2-small MLP forward: M=16384 (8x2048), d=768, h=3072"),
    "step16k": Workload(
        "step16k", M=16384, d=768, h=3072,
        description="GPT-2-small MLP fwd+bwd step: M=16384 (8x2048), d=768, h=3072"),
    "train49k": Workload(
        "train49k", M=49152, d=768, h=3072, steps=20, perturb_var=1e-3,
        description="GPT-2-small MLP train step: M=49152 (48x1024), d=768, "
                    "h=3072, 20 steps, W += N(0,1e-3), W2 cache refreshed per step"),
    "stack9": Workload(
        "stack9", M=131072, d=768, h=3072, layers=9,
        description="9-layer stack of 768-dim ReLU^2 MLP blocks, M=131072 "
                    "(64x2048), BF16 residual r0~N(0,1), per-layer RMSNorm"),
    "qkv16k": Workload(
        "qkv16k", M=16384, d=768, h=2304,
        description="FP8 linear layer y = x W^T as the attention QKV projection: M=16384 tokens, "
                    "K=768, N=2304 (3x768), e4m3 forward, BF16 backward"),
    "ce16k": Workload(
        "ce16k", M=16384, d=768, h=50304,
        description="softcapped cross-entropy over a GPT-2 LM head: M=16384 tokens, d=768, "
                    "V=50304 (GPT-2 vocabulary padded to a multiple of 128), logits std 4, "
                    "cap 15, one uniform target per token, fwd + bwd (dlogits, dX, dW)"),
    "heavytail": Workload(
        "heavytail", M=65536, d=1024, h=4096, steps=30, x_dist="student_t3",
        spike_steps=(9, 19, 29), spike_factor=2.0,
        description="M=65536 d=1024 h=4096, x~Student-t(3) clipped to +-64, "
                    "30 steps, x*2 (post*4) at 0-based steps 9, 19, 29"),
}


def _normal(g, shape, var):
    return g.standard_normal(shape, dtype=np.float32) * np.float32(np.sqrt(var))


def _grid(g, shape, k, denom):
    return g.integers(-k, k + 1, size=shape).astype(np.float32) / np.float32(denom)


def make_x(g, M, d, dist):
    if dist == "normal":
        return _normal(g, (M, d), 1.0)
    if dist == "student_t3":
        return np.clip(g.standard_t(3, size=(M, d)), -64, 64).astype(np.float32)
    if dist == "grid":
        return _grid(g, (M, d), 8, 4)           # k/4, |k| <= 8
    raise ValueError(dist)


def make_w(g, rows, cols, var, dist):
    if dist == "normal":
        return _normal(g, (rows, cols), var)
    if dist == "grid":
        return _grid(g, (rows, cols), 16, 256)  # k/256, |k| <= 16
    raise ValueError(dist)


def make_problem(M, d, h, seed=0, x_dist="normal", w_dist="normal"):
    """One MLP problem: x [M,d], W1 [h,d], W2 [h,d], dOut [M,d] as BF16 bits."""
    g = rng(seed)
    W1 = make_w(g, h, d, 1.0 / d, w_dist)
    W2 = make_w(g, h, d, 1.0 / h, w_dist)
    x = make_x(g, M, d, x_dist)
    dOut = make_x(g, M, d, "grid" if x_dist == "grid" else "normal")
    return dict(x=to_bf16_bits(x), W1=to_bf16_bits(W1), W2=to_bf16_bits(W2),
                dOut=to_bf16_bits(dOut))


def make_head_problem(M, d, V, T=1, seed=0, x_dist="normal", logit_std=4.0, ignore_frac=0.0):
    """One LM-head problem: x [M,d] and W [V,d] as BF16 bits, targets [M,T]
    int32 uniform in [0, V), a fraction ``ignore_frac`` of them set to -1.

    W ~ N(0, logit_std^2 / d) gives logits of standard deviation about
    logit_std for x ~ N(0, 1); ``grid`` draws x = k/4, W = k/256."""
    g = rng(seed)
    if x_dist == "grid":
        x = _grid(g, (M, d), 8, 4)
        W = _grid(g, (V, d), 16, 256)
    else:
        x = make_x(g, M, d, x_dist)
        W = _normal(g, (V, d), logit_std ** 2 / d)
    tg = g.integers(0, V, size=(M, T)).astype(np.int32)
    if ignore_frac > 0:
        tg[g.random((M, T)) < ignore_frac] = -1
    return dict(x=to_bf16_bits(x), W=to_bf16_bits(W), targets=tg)


def perturb(W_bits, seed, step, var, which):
    """W + N(0, var) drawn from seed + 1000*step (+1 for W2), rounded to BF16."""
    g = rng(seed + 1000 * step + (1 if which == "W2" else 0))
    W = torch.from_numpy(W_bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    return to_bf16_bits(W + _normal(g, W.shape, var))


def make_partials(n, seed=0, scale=1.0):
    """Synthetic partial-amax values (non-negative fp32) for the scale update."""
    g = rng(seed)
    return (np.abs(g.standard_normal(n)) * scale).astype(np.float32)
