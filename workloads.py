"""Seeded synthetic BF16 inputs shaped like the models the formats were tested on.

This module only draws random tensors; it contains none of the quantisation
arithmetic, so the GPU library and the CPU oracle can both be fed from it.

Shapes follow the model families named on "Low Precision RL" ("Choose a
precision": Qwen3-4B, Qwen3-30B-A3B, DeepSeek-V3 for FP8 block-wise,
Qwen3-30B-A3B for MXFP8) and the verl NVFP4 QAT article (section 2.4: q/k/v
and gate/up fusion siblings; section 2.3: W4A16 weights, W4A4 activations).

Recipe: seed = workload index * 1000 + tensor index; values drawn in FP32
(normal with the stated standard deviation) and rounded to BF16 with
round-to-nearest-even by torch; outliers are multiplied into a seeded choice
of positions without replacement.  Small workloads are drawn on the CPU;
large ones on the device the caller passes (torch's CUDA generator), and any
oracle check of them copies the very same bytes back to the host.
"""
from dataclasses import dataclass, field
import math
from typing import List, Optional, Tuple

import torch


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal_bf16(shape, std: float, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    x.mul_(std)
    return x.to(torch.bfloat16)


def with_outliers(x: torch.Tensor, frac: float, factor: float, seed: int) -> torch.Tensor:
    """Multiply round(frac * numel) seeded positions (no replacement) by factor."""
    n = x.numel()
    k = int(round(frac * n))
    if k == 0:
        return x
    g = _gen(seed + 500, "cpu")
    idx = torch.randperm(n, generator=g)[:k].to(x.device)
    flat = x.view(-1)
    flat[idx] = (flat[idx].float() * factor).to(torch.bfloat16)
    return x


def outlier_channels(x: torch.Tensor, n_channels: int, factor: float, seed: int) -> torch.Tensor:
    """Multiply n_channels seeded columns of the last dimension by factor."""
    g = _gen(seed + 700, "cpu")
    cols = torch.randperm(x.shape[-1], generator=g)[:n_channels].to(x.device)
    x[..., cols] = (x[..., cols].float() * factor).to(torch.bfloat16)
    return x


# ------------------------------------------------------------------ shapes

QWEN3_4B_LAYER: List[Tuple[str, Tuple[int, int]]] = [
    ("q_proj", (4096, 2560)), ("k_proj", (1024, 2560)), ("v_proj", (1024, 2560)),
    ("o_proj", (2560, 4096)), ("gate_proj", (9728, 2560)), ("up_proj", (9728, 2560)),
    ("down_proj", (2560, 9728)),
]
QWEN3_4B_LAYERS = 36
# NVFP4 sibling groups of a dense decoder layer (names index QWEN3_4B_LAYER)
QWEN3_4B_GROUPS = [("q_proj", "k_proj", "v_proj"), ("o_proj",), ("gate_proj", "up_proj"),
                   ("down_proj",)]

QWEN3_30B_EXPERTS = 128
QWEN3_30B_EXPERT_SHAPES = [("gate", (768, 2048)), ("up", (768, 2048)), ("down", (2048, 768))]
QWEN3_30B_LAYERS = 48

BLOCK2048_TENSORS = [("q_proj", (4096, 2048)), ("k_proj", (512, 2048)), ("v_proj", (512, 2048)),
                     ("gate_proj", (6144, 2048)), ("up_proj", (6144, 2048)),
                     ("down_proj", (2048, 6144))]
BLOCK2048_GROUPS = [("q_proj", "k_proj", "v_proj"), ("gate_proj", "up_proj"), ("down_proj",)]

DSV3_EXPERTS = 256
DSV3_EXPERT_SHAPES = [("gate", (2048, 7168)), ("up", (2048, 7168)), ("down", (7168, 2048))]
DSV3_ACT_SHAPE = (16384, 7168)


# ------------------------------------------------------------------ workloads

def small_matrix(device="cpu") -> torch.Tensor:
    """256 x 512, N(0, 0.02), 0.1% of entries (131) multiplied by 50."""
    x = normal_bf16((256, 512), 0.02, seed=1000, device=device)
    return with_outliers(x, 131 / (256 * 512), 50.0, seed=1000)


def qwen3_4b_layer(layer: int, device="cpu") -> dict:
    """One decoder layer of Qwen3-4B-shaped dense weights, N(0, 0.02)."""
    out = {}
    for t, (name, shape) in enumerate(QWEN3_4B_LAYER):
        out[name] = normal_bf16(shape, 0.02, seed=2000 + layer * len(QWEN3_4B_LAYER) + t,
                                device=device)
    return out


def qwen3_30b_moe_layer(layer: int, device="cpu", experts: int = QWEN3_30B_EXPERTS) -> dict:
    """Batched experts [E][rows][cols], N(0, 0.02) times a per-expert factor
    drawn from LogUniform(0.5, 2)."""
    g = _gen(3000 + layer * 10 + 9, "cpu")
    u = torch.rand(experts, generator=g, dtype=torch.float64)
    factor = torch.exp(math.log(0.5) + u * (math.log(2.0) - math.log(0.5)))
    out = {}
    for t, (name, (r, c)) in enumerate(QWEN3_30B_EXPERT_SHAPES):
        g2 = _gen(3000 + layer * 10 + t, device)
        x = torch.randn((experts, r, c), generator=g2, device=device, dtype=torch.float32)
        x.mul_(0.02 * factor.to(device=device, dtype=torch.float32).view(-1, 1, 1))
        out[name] = x.to(torch.bfloat16)
    return out


def block2048(device="cpu") -> dict:
    """2048-hidden block: q/k/v and gate/up siblings plus down, N(0, 0.02)
    with 0.05% of entries multiplied by 100."""
    out = {}
    for t, (name, shape) in enumerate(BLOCK2048_TENSORS):
        x = normal_bf16(shape, 0.02, seed=4000 + t, device=device)
        out[name] = with_outliers(x, 0.0005, 100.0, seed=4000 + t)
    return out


def block2048_grad(name: str, device="cpu") -> torch.Tensor:
    """Upstream gradient for the straight-through backward, N(0, 1) * 1e-3."""
    shape = dict(BLOCK2048_TENSORS)[name]
    return normal_bf16(shape, 1e-3, seed=4100 + [n for n, _ in BLOCK2048_TENSORS].index(name),
                       device=device)


def dsv3_experts(device="cpu", experts: int = DSV3_EXPERTS, seed: int = 5000) -> dict:
    """DeepSeek-V3-shaped routed experts, batched [E][rows][cols], N(0, 0.01)."""
    out = {}
    for t, (name, (r, c)) in enumerate(DSV3_EXPERT_SHAPES):
        out[name] = normal_bf16((experts, r, c), 0.01, seed=seed + t, device=device)
    return out


def dsv3_activation(device="cpu", seed: int = 5100) -> torch.Tensor:
    """16384 x 7168 activation, N(0, 1) with 8 seeded channels multiplied by 20."""
    x = normal_bf16(DSV3_ACT_SHAPE, 1.0, seed=seed, device=device)
    return outlier_channels(x, 8, 20.0, seed=seed)


def random_bf16(shape, seed: int, std: float = 1.0, device="cpu") -> torch.Tensor:
    return normal_bf16(shape, std, seed=seed, device=device)


def random_code_bytes(shape, seed: int, max_mag: int, device="cpu") -> torch.Tensor:
    """Uniform random 8-bit code bytes: low seven bits 0..max_mag, random top
    (sign) bit; uint8."""
    g = _gen(seed, device)
    mag = torch.randint(0, max_mag + 1, shape, generator=g, device=device, dtype=torch.uint8)
    sign = torch.randint(0, 2, shape, generator=g, device=device, dtype=torch.uint8)
    return mag | (sign << 7)


def bits(x: torch.Tensor):
    """BF16 tensor -> numpy uint16 bit patterns (host copy)."""
    return x.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")


def from_bits(b, device="cpu") -> torch.Tensor:
    import numpy as np
    t = torch.from_numpy(np.ascontiguousarray(b).view(np.int16).copy())
    return t.view(torch.bfloat16).to(device)
