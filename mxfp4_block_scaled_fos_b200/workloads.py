"""Seeded synthetic inputs for the quantizer (no quantization arithmetic here).

This module only draws random tensors.  The CUDA path and the CPU reference
used by the tests receive the same bf16 bytes from it, so it holds none of the
method's arithmetic.  Every recipe follows the workload descriptions of the
Four Over Six / FP4 pages' use cases (activations with outlier channels,
weights, gradients, MoE expert weights) and the worked example of the
Ultralytics "FP4" glossary page ("Como funciona FP4": ``torch.randn(4096)``
under seed 0 with every 512th value scaled by 20).

Sizes are parameters so tests can use the same recipe at small sizes; the
default sizes are the full workloads.
"""
from __future__ import annotations

import torch

# name -> (batch, rows, cols) at full size
FULL_SHAPES = {
    "outlier_vector": (1, 128, 256),
    "activation_outliers": (1, 8192, 4096),
    "weight_normal": (1, 14336, 4096),
    "gradient_student_t": (1, 16384, 8192),
    "moe_experts": (128, 2880, 2880),
}


def page_example_input() -> torch.Tensor:
    """The worked example's fp32 input: seed 0, randn(4096), x[::512] *= 20."""
    torch.manual_seed(0)
    x = torch.randn(4096)
    x[::512] *= 20
    return x


def outlier_vector(rows: int = 128, cols: int = 256) -> torch.Tensor:
    """The worked example's generator pattern at rows*cols values (CPU)."""
    torch.manual_seed(0)
    x = torch.randn(rows * cols)
    x[::512] *= 20
    return x.to(torch.bfloat16).view(1, rows, cols)


def activation_outliers(rows: int = 8192, cols: int = 4096, device="cpu",
                        seed: int = 0, frac: float = 0.01, gain: float = 50.0) -> torch.Tensor:
    """N(0,1) rows with round(frac*cols) seeded outlier channels scaled by gain."""
    g = torch.Generator(device=device).manual_seed(seed)
    x = torch.randn(rows, cols, generator=g, device=device)
    n_out = max(1, round(frac * cols))
    cols_idx = torch.randperm(cols, generator=torch.Generator().manual_seed(seed + 1))[:n_out]
    x[:, cols_idx.to(device)] *= gain
    return x.to(torch.bfloat16).view(1, rows, cols)


def weight_normal(rows: int = 14336, cols: int = 4096, device="cpu", seed: int = 0,
                  std: float = 0.02) -> torch.Tensor:
    g = torch.Generator(device=device).manual_seed(seed)
    x = torch.randn(rows, cols, generator=g, device=device) * std
    return x.to(torch.bfloat16).view(1, rows, cols)


def gradient_student_t(rows: int = 16384, cols: int = 8192, device="cpu", seed: int = 0,
                       scale: float = 1e-3) -> torch.Tensor:
    """Student-t with 3 degrees of freedom: Z / sqrt((Z1^2+Z2^2+Z3^2)/3), times scale."""
    g = torch.Generator(device=device).manual_seed(seed)
    z = torch.randn(rows, cols, generator=g, device=device)
    chi = torch.zeros_like(z)
    for _ in range(3):
        zi = torch.randn(rows, cols, generator=g, device=device)
        chi.addcmul_(zi, zi)
        del zi
    x = z / torch.sqrt(chi / 3.0) * scale
    del z, chi
    return x.to(torch.bfloat16).view(1, rows, cols)


def moe_experts(experts: int = 128, rows: int = 2880, cols: int = 2880, device="cpu",
                seed: int = 0, std: float = 0.02) -> torch.Tensor:
    """Per-expert N(0, std^2) times s_e ~ U(0.5, 2), drawn expert by expert."""
    gs = torch.Generator().manual_seed(seed)
    s_e = 0.5 + 1.5 * torch.rand(experts, generator=gs)
    g = torch.Generator(device=device).manual_seed(seed)
    out = torch.empty(experts, rows, cols, dtype=torch.bfloat16, device=device)
    for e in range(experts):
        w = torch.randn(rows, cols, generator=g, device=device)
        out[e] = (w * (std * float(s_e[e]))).to(torch.bfloat16)
    return out


def make(name: str, device="cpu", shape=None, seed: int = 0) -> torch.Tensor:
    """Build a named workload as a [batch, rows, cols] bf16 tensor."""
    b, r, c = shape if shape is not None else FULL_SHAPES[name]
    if name == "outlier_vector":
        return outlier_vector(r, c).to(device)
    if name == "activation_outliers":
        return activation_outliers(r, c, device=device, seed=seed)
    if name == "weight_normal":
        return weight_normal(r, c, device=device, seed=seed)
    if name == "gradient_student_t":
        return gradient_student_t(r, c, device=device, seed=seed)
    if name == "moe_experts":
        return moe_experts(b, r, c, device=device, seed=seed)
    raise KeyError(name)


def bits(x: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    return x.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")
