"""Seeded synthetic inputs shared by the CUDA path's tests, the bench and the oracle.

This module only draws random numbers and names shapes: it holds none of the
quantization or LoRA arithmetic, so both sides of every parity check can take
their inputs from it.

Shapes follow the pages' workloads: OPT-1.3B decoder linears (d_model 2048,
24 layers, fc 8192; "FT-02: QLoRA -- Fine-Tuning with Quantization", guided
example 3) and a 7B decoder layer with d = 4096, FFN 14336 and 32 query / 8
key-value heads of 128 ("QLoRA: NF4 storage, gradients and local
integration", section "Memory accounting before optimization").  Their
checkpoints are not available; Gaussian weights of the stated scale stand in.

Distributions: weights N(0, 0.02) (standard deviation), optionally with a
0.1% Bernoulli mask of entries multiplied by 10 ("outliers"); activations and
upstream gradients N(0, 1) drawn in fp32 and rounded to bf16; LoRA matrices as
each configuration states.  Seeds: ``1000 * config + 10 * layer + tensor``
for weights, with fixed offsets for the other tensor families.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import torch

W_STD = 0.02
OUTLIER_FRAC = 0.001
OUTLIER_SCALE = 10.0

SEED_A = 100_000
SEED_B = 200_000
SEED_X = 300_000
SEED_DY = 400_000


def weight_seed(config: int, layer: int, tensor: int) -> int:
    return 1000 * config + 10 * layer + tensor


def normal_f32(shape, std: float, seed: int, device="cpu") -> torch.Tensor:
    """fp32 N(0, std^2) samples from a seeded torch generator on ``device``."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return torch.randn(tuple(shape), generator=g, dtype=torch.float32, device=device) * float(std)


def with_outliers(w: torch.Tensor, seed: int, frac: float = OUTLIER_FRAC, scale: float = OUTLIER_SCALE) -> torch.Tensor:
    """Multiply a seeded Bernoulli(frac) subset of entries by ``scale`` (in place)."""
    g = torch.Generator(device=w.device)
    g.manual_seed(int(seed) + 7_777_777)
    mask = torch.rand(w.shape, generator=g, device=w.device) < frac
    w[mask] *= scale
    return w


def normal_bf16(shape, std: float, seed: int, device="cpu") -> torch.Tensor:
    """N(0, std^2) drawn in fp32, then rounded to bf16 (nearest even)."""
    return normal_f32(shape, std, seed, device).to(torch.bfloat16)


# ---------------------------------------------------------------------------
# Configurations
# ---------------------------------------------------------------------------

@dataclass
class Projection:
    name: str
    n: int  # d_out (rows of W0)
    k: int  # d_in  (cols of W0)


OPT13B_LAYER = [
    Projection("q", 2048, 2048),
    Projection("k", 2048, 2048),
    Projection("v", 2048, 2048),
    Projection("o", 2048, 2048),
    Projection("fc1", 8192, 2048),
    Projection("fc2", 2048, 8192),
]
OPT13B_LAYERS = 24

LAYER7B = [
    Projection("q", 4096, 4096),
    Projection("k", 1024, 4096),
    Projection("v", 1024, 4096),
    Projection("o", 4096, 4096),
    Projection("gate", 14336, 4096),
    Projection("up", 14336, 4096),
    Projection("down", 4096, 14336),
]
LAYERS7B = 32

GATE7B = Projection("gate", 14336, 4096)


def opt13b_weight_shapes():
    """(layer, tensor index, Projection) for the 168 OPT-1.3B-shaped tensors."""
    return [(layer, t, p) for layer in range(OPT13B_LAYERS) for t, p in enumerate(OPT13B_LAYER)]


def opt13b_weight(layer: int, t: int, device="cpu") -> torch.Tensor:
    p = OPT13B_LAYER[t]
    w = normal_f32((p.n, p.k), W_STD, weight_seed(2, layer, t), device)
    return with_outliers(w, weight_seed(2, layer, t))


@dataclass
class TinyCase:
    W: torch.Tensor  # fp32 [1024, 1024], block 0 all zeros
    A: torch.Tensor  # bf16 [8, 1024]
    B: torch.Tensor  # bf16 [1024, 8]
    X: torch.Tensor  # bf16 [16, 1024]
    dY: torch.Tensor  # bf16 [16, 1024]
    r: int = 8
    alpha: float = 16.0

    @property
    def s(self) -> float:
        return self.alpha / self.r


def tiny_case() -> TinyCase:
    """1024x1024 weight N(0, 0.02) (seed 0) with its first 64-block zeroed;
    r = 8, alpha = 16; A ~ N(0, (1/8)^2), B ~ N(0, 0.01^2); X, dY 16 x 1024 ~ N(0, 1)."""
    W = normal_f32((1024, 1024), W_STD, 0)
    W[0, :64] = 0.0
    A = normal_bf16((8, 1024), 1.0 / 8.0, 1)
    B = normal_bf16((1024, 8), 0.01, 2)
    X = normal_bf16((16, 1024), 1.0, 3)
    dY = normal_bf16((16, 1024), 1.0, 4)
    return TinyCase(W, A, B, X, dY)


@dataclass
class LinearCase:
    """One adapted projection: weight, adapters and a batch of activations."""

    proj: Projection
    W: torch.Tensor
    A: torch.Tensor
    B: torch.Tensor
    X: torch.Tensor
    dY: torch.Tensor | None
    r: int
    alpha: float
    extra: dict = field(default_factory=dict)

    @property
    def s(self) -> float:
        return self.alpha / self.r


def linear_case(proj: Projection, m: int, r: int, alpha: float, config: int, layer: int, t: int,
                device="cpu", ab_std: float = 0.02, outliers: bool = False, with_dy: bool = True) -> LinearCase:
    """Seeded inputs of one projection of configuration ``config``."""
    seed = weight_seed(config, layer, t)
    W = normal_f32((proj.n, proj.k), W_STD, seed, device)
    if outliers:
        with_outliers(W, seed)
    A = normal_bf16((r, proj.k), ab_std, SEED_A + seed, device)
    B = normal_bf16((proj.n, r), ab_std, SEED_B + seed, device)
    X = normal_bf16((m, proj.k), 1.0, SEED_X + seed, device)
    dY = normal_bf16((m, proj.n), 1.0, SEED_DY + seed, device) if with_dy else None
    return LinearCase(proj, W, A, B, X, dY, r, alpha)


def gemv_case(m: int, device="cpu") -> LinearCase:
    """Decode-shaped gate projection 14336 x 4096, r = 16, alpha = 32, A, B ~ N(0, 0.02^2)."""
    return linear_case(GATE7B, m, 16, 32.0, 3, 0, 4, device, with_dy=False)


def layer7b_case(t: int, m: int = 8192, device="cpu", layer: int = 0, config: int = 4,
                 outliers: bool = False) -> LinearCase:
    """Projection ``t`` of the training-shaped 7B layer at ``m`` tokens, r = 16, alpha = 32."""
    return linear_case(LAYER7B[t], m, 16, 32.0, config, layer, t, device, outliers=outliers)


# ---------------------------------------------------------------------------
# 32-layer stack of the 7B layer's projections (weights with 0.1% outliers)
# ---------------------------------------------------------------------------

STACK_CONFIG = 5


def stack_projection(layer: int, t: int, device="cpu", r: int = 16, ab_std: float = 0.02):
    """(W fp32, A bf16, B bf16) of projection ``t`` of stack layer ``layer``."""
    p = LAYER7B[t]
    seed = weight_seed(STACK_CONFIG, layer, t)
    W = with_outliers(normal_f32((p.n, p.k), W_STD, seed, device), seed)
    A = normal_bf16((r, p.k), ab_std, SEED_A + seed, device)
    B = normal_bf16((p.n, r), ab_std, SEED_B + seed, device)
    return W, A, B


def stack_input(m: int, device="cpu") -> torch.Tensor:
    """The stack's input activations h_0, bf16 [m, 4096] ~ N(0, 1)."""
    return normal_bf16((m, 4096), 1.0, SEED_X + weight_seed(STACK_CONFIG, 99, 0), device)


def stack_leaf_grad(layer: int, which: str, m: int, device="cpu") -> torch.Tensor:
    """Seeded upstream gradients: the k and v outputs of each layer are leaves
    ("k", "v": [m, 1024]); "top" is the gradient of the last layer's output [m, 4096]."""
    cols = {"k": 1024, "v": 1024, "top": 4096}[which]
    idx = {"k": 1, "v": 2, "top": 7}[which]
    return normal_bf16((m, cols), 1.0, SEED_DY + weight_seed(STACK_CONFIG, layer, idx), device)
