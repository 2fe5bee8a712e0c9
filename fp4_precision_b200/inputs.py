"""Seeded synthetic workloads for the FP4 quantized linear layer.

This module only draws random tensors; it holds none of the method's
arithmetic, and both the CUDA path's tests/benchmark and the CPU oracle's tests
use it. The shapes stand in for the layers the pages train (Llama-3.1-8B on C4
in "New AMD paper overturns conventional wisdom: FP4 training...", section
"Poiskovaya eksperimental'naya rabota"); no dataset or checkpoint is used.

Every tensor comes from its own ``torch.Generator`` seeded from (workload seed,
tensor name), so a tensor is the same whatever else is drawn, on a given device.
A generator on a CUDA device draws different numbers than one on the CPU; the
tests that compare the two paths copy the same bf16 bytes to both sides.
"""
from __future__ import annotations

import zlib

import torch

__all__ = ["normal", "normal_with_outliers", "student_t_colgain", "silu_product", "workload", "WORKLOADS"]


def _gen(seed: int, name: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + zlib.crc32(name.encode())) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def normal(shape, std: float, seed: int, name: str, device="cpu") -> torch.Tensor:
    """N(0, std^2) in bf16."""
    g = _gen(seed, name, device)
    return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)


def normal_with_outliers(shape, seed: int, name: str, device="cpu", frac: float = 1e-3,
                         factor: float = 50.0) -> torch.Tensor:
    """N(0, 1) with a Bernoulli(frac) mask of entries multiplied by ``factor``."""
    g = _gen(seed, name, device)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    mask = torch.rand(shape, generator=g, device=device) < frac
    x = torch.where(mask, x * factor, x)
    return x.to(torch.bfloat16)


def student_t_colgain(shape, seed: int, name: str, device="cpu", nu: int = 3, scale: float = 0.02) -> torch.Tensor:
    """Student-t(nu) * scale * g_col with per-column gains g_col ~ LogNormal(0, 1).
    t = z0 / sqrt(chi2_nu / nu), chi2_nu a sum of nu squared standard normals."""
    g = _gen(seed, name, device)
    R, C = shape
    z0 = torch.randn((R, C), generator=g, device=device)
    chi2 = torch.zeros((R, C), device=device)
    for _ in range(nu):
        z = torch.randn((R, C), generator=g, device=device)
        chi2 += z * z
    t = z0 / torch.sqrt(chi2 / nu)
    gain = torch.exp(torch.randn((1, C), generator=g, device=device))
    return (t * scale * gain).to(torch.bfloat16)


def silu_product(shape, seed: int, name: str, device="cpu") -> torch.Tensor:
    """SiLU(N(0,1)) * N(0,1): the input of an MLP down projection."""
    g = _gen(seed, name, device)
    a = torch.randn(shape, generator=g, device=device)
    b = torch.randn(shape, generator=g, device=device)
    return (torch.nn.functional.silu(a) * b).to(torch.bfloat16)


# name -> (description, M, N, K, seed)
WORKLOADS = {
    "tiny": ("tiny NVFP4 linear: X [512x256], W [256x256], dY [512x256], N(0,1) + 0.1% x50 outliers", 512, 256, 256, 0),
    "sweep": ("quantizer sweep tensor [8192x4096], Student-t(3)*0.02*LogNormal(0,1) column gains", 8192, 0, 4096, 1),
    "qkv": ("Llama-3.1-8B QKV projection: X [8192x4096], W [6144x4096], dY [8192x6144]", 8192, 6144, 4096, 2),
    "mlp_up": ("Llama-3.1-8B MLP up/gate: X [16384x4096], W [28672x4096], dY [16384x28672]", 16384, 28672, 4096, 3),
    "mlp_down": ("Llama-3.1-8B MLP down: X [Mx14336] = SiLU(N)*N, W [4096x14336], dY [Mx4096]", 16384, 4096, 14336, 4),
}


def workload(name: str, device="cpu", M: int | None = None) -> dict:
    """Tensors of a named workload. Linear workloads return X [M,K], W [N,K] and
    dY [M,N] in bf16; the quantizer sweep returns T [8192, 4096]."""
    desc, M0, N, K, seed = WORKLOADS[name]
    M = M0 if M is None else M
    if name == "sweep":
        return {"T": student_t_colgain((M, K), seed, "T", device)}
    if name == "tiny":
        return {"X": normal_with_outliers((M, K), seed, "X", device),
                "W": normal_with_outliers((N, K), seed, "W", device),
                "dY": normal_with_outliers((M, N), seed, "dY", device)}
    if name == "mlp_down":
        X = silu_product((M, K), seed, "X", device)
    else:
        X = normal_with_outliers((M, K), seed, "X", device)
    return {"X": X, "W": normal((N, K), 0.02, seed, "W", device), "dY": normal((M, N), 1e-3, seed, "dY", device)}
